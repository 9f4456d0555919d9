"""include/q4k.h from plain C: a C99 program compiled with gcc against the
header and linked with libq4k_b200.so, run on the CPU (it makes only calls the
library answers on the host)."""
import os
import shutil
import subprocess

import pytest

from gguf_quant_dequant_q4k_b200 import capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_compiles_as_c99_and_links(tmp_path):
    exe = os.path.join(tmp_path, "abi_check")
    libdir = os.path.dirname(capi.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi", "abi_check.c"),
           "-L", libdir, "-l:" + os.path.basename(capi.LIB_PATH),
           "-Wl,-rpath," + libdir, "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "c abi check ok" in r.stdout
