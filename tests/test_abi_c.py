"""include/qlora.h is a plain C header: a C99 program compiled with gcc
(-pedantic, warnings as errors) includes it, takes the address of every entry
point, links against the built library and runs its host-only checks (sizes,
codebook, argument errors, status names); the binding's ctypes structs are
compared with the C layout it prints. No kernel is launched."""

import ctypes
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_client(lib, tmp_path):
    so = lib.library_path
    exe = tmp_path / "abi_check"
    cmd = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_c", "abi_check.c"),
           "-o", str(exe), so, "-Wl,-rpath," + os.path.dirname(so)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    lines = run.stdout.strip().splitlines()
    assert run.returncode == 0 and lines[-1] == "ok", run.stdout + run.stderr
    return lines


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_compiles_as_c99_and_links(lib, tmp_path):
    _run_client(lib, tmp_path)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_binding_structs_match_the_c_layout(lib, tmp_path):
    """The ctypes mirrors of the header's structs have the C compiler's size
    and field offsets."""
    from bit_nf4_quantized_dequant_b200 import _binding as b
    mirrors = {"qlora_nf4_t": b._NF4, "qlora_linear_problem_t": b._Problem, "qlora_adamw8_tensor_t": b._Adam8}
    seen = set()
    for line in _run_client(lib, tmp_path):
        if not line.startswith("layout "):
            continue
        _, name, size, *fields = line.split()
        cls = mirrors[name]
        assert ctypes.sizeof(cls) == int(size), name
        for f in fields:
            field, off = f.split("=")
            assert getattr(cls, field).offset == int(off), (name, field)
        assert [f for f, _ in cls._fields_] == [f.split("=")[0] for f in fields], name
        seen.add(name)
    assert seen == set(mirrors)


def test_every_entry_point_is_in_the_c_client():
    """The C client's table names every function the header declares."""
    from test_abi import declared_symbols
    text = open(os.path.join(ROOT, "tests", "abi_c", "abi_check.c")).read()
    missing = [s for s in declared_symbols() if f"(any_fn){s}" not in text]
    assert not missing, missing
