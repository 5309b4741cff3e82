"""The C ABI from plain C: compile tests/c/abi_consumer.c with gcc against the
headers in include/, link it to the built shared library and run its
host-only checks (no GPU, no device work)."""

import os
import shutil
import subprocess

import pytest

import bit_nf4_quantized_26_b200 as q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_plain_c_consumer():
    src = os.path.join(ROOT, "tests", "c", "abi_consumer.c")
    libdir = os.path.dirname(q.LIB_PATH)
    outdir = os.path.join(libdir, "_build")  # the library's (untracked) build folder
    os.makedirs(outdir, exist_ok=True)
    exe = os.path.join(outdir, "abi_consumer")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src, "-o", exe,
                    "-L", libdir, "-lqlora_nf4", "-Wl,-rpath," + libdir, "-lm"], check=True)
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    assert "c abi consumer ok" in out.stdout
