"""include/qlora.h is a plain C header: a C99 program compiled with gcc
(-pedantic, warnings as errors) includes it, takes the address of every entry
point, links against the built library and runs its host-only checks (sizes,
codebook, argument errors, status names). No kernel is launched."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_compiles_as_c99_and_links(lib, tmp_path):
    so = lib.library_path
    exe = tmp_path / "abi_check"
    cmd = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_c", "abi_check.c"),
           "-o", str(exe), so, "-Wl,-rpath," + os.path.dirname(so)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr


def test_every_entry_point_is_in_the_c_client():
    """The C client's table names every function the header declares."""
    from test_abi import declared_symbols
    text = open(os.path.join(ROOT, "tests", "abi_c", "abi_check.c")).read()
    missing = [s for s in declared_symbols() if f"(any_fn){s}" not in text]
    assert not missing, missing
