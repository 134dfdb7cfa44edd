"""ctypes binding of libqlora (filled in with the C ABI)."""

__all__ = []
