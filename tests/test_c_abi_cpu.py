"""The C ABI from plain C99 on the host: tests/c_abi/abi_host.c is compiled
against include/dsa.h (-std=c99 -pedantic -Werror), linked to the in-tree
libdsa.so with no Python or torch in the process, and run; it checks the
calls that need no device (see its header)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_attention_decode_lightning_b200")


def test_host_calls_from_plain_c(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    if not os.path.exists(os.path.join(PKG, "libdsa.so")):
        pytest.skip("libdsa.so is not built")
    exe = str(tmp_path / "abi_host")
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi", "abi_host.c"),
                    "-L", PKG, "-ldsa", "-Wl,-rpath," + PKG, "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "host calls ok" in r.stdout
