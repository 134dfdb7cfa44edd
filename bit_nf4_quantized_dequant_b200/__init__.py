"""libqlora: the NF4 QLoRA linear layer on one B200 (sm_100a).

The compute path lives in the C-ABI shared library ``libqlora.so`` built from
``csrc/`` (see ``include/qlora.h``); this package is a thin ctypes binding
that marshals torch device tensors into the C calls. The library is loaded on
first use; if it is missing or fails to load, every call raises.
"""

from ._binding import *  # noqa: F401,F403
from ._binding import __all__  # noqa: F401
