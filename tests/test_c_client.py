"""The C ABI from plain C: tests/c/abi_host.c, a C99 program that includes
only include/gradsolve.h and links libgradsolve.so, compiles with warnings as
errors and passes its host-side checks (status strings, workspace sizes,
argument validation, the empty ensemble).  No GPU work."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "discrete_adjoint_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_client(tmp_path):
    import discrete_adjoint_b200  # noqa: F401  (fails here if the library has not been built)
    exe = str(tmp_path / "abi_host")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"), "-L", LIBDIR, "-lgradsolve",
                    "-Wl,-rpath," + LIBDIR, "-o", exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
