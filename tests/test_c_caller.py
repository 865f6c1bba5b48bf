"""The C ABI from a plain C99 program (no GPU needed): include/attnqat.h
compiles as C, libattnqat.so links, and the host-side checks return the
documented status codes."""
import os
import shutil
import subprocess

import pytest

import quantization_aware_attention_nvfp4_b200 as A
from quantization_aware_attention_nvfp4_b200 import build as B

HERE = os.path.dirname(os.path.abspath(__file__))


def test_c99_caller_builds_links_and_validates(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    A.load()  # builds the library if it is missing or stale
    lib = B.LIB
    exe = str(tmp_path / "abi_from_c")
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Werror", "-I" + B.INCLUDE, os.path.join(HERE, "c", "abi_from_c.c"),
                           lib, "-Wl,-rpath," + os.path.dirname(lib), "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
