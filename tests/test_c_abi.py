"""The boundary is a C ABI, not only a ctypes surface: a plain C99 program
(tests/c_abi_check.c) includes the header, links against libtri_attn.so and
checks the host-side answers of the attention, triangle-multiplication and
projection entry points. No GPU: every call it makes fails (as it must) before
any CUDA work."""

import os
import shutil
import subprocess

import pytest

import triangle_attention_b200 as ta
from triangle_attention_b200 import build as tbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_links_and_checks(tmp_path):
    tbuild.build()
    libdir = os.path.dirname(ta.LIB_PATH)
    exe = tmp_path / "c_abi_check"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c_abi_check.c"),
                           "-L", libdir, "-l:libtri_attn.so", f"-Wl,-rpath,{libdir}",
                           "-o", str(exe)])
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr
    assert "c abi ok" in res.stdout
