"""The C ABI from C: tests/c_consumer.c is compiled as strict C99 (-pedantic,
warnings as errors) against include/dsa.h, linked against the built
libdsa.so, and run.  It exercises only host-side refusals and workspace
queries, so it needs no GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_attention_13_b200")
OUT = os.path.join(ROOT, "build", "c_consumer")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_uses_the_abi():
    if not os.path.exists(os.path.join(PKG, "libdsa.so")):
        pytest.skip("libdsa.so not built")
    os.makedirs(OUT, exist_ok=True)
    exe = os.path.join(OUT, "c_consumer")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_consumer.c"),
                    "-L", PKG, "-ldsa", f"-Wl,-rpath,{PKG}", "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, f"check {r.returncode} failed: {r.stderr}"
    assert r.stdout.strip() == "ok"
