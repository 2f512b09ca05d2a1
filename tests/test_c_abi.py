"""The boundary is plain C: a C99 program that includes only
include/nf4lora.h compiles with gcc (-Wall -Werror), links against the built
libnf4lora.so and runs its host-only checks (sizing, buffer layout, argument
validation) without a GPU."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "nf4_base_lora_b200", "lib")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_caller_compiles_links_and_runs():
    assert os.path.exists(os.path.join(LIB_DIR, "libnf4lora.so")), "build the library first"
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "abi_check")
        subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_check.c"),
                        "-L", LIB_DIR, "-lnf4lora", "-Wl,-rpath," + LIB_DIR, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert out.returncode == 0, out.stderr
        assert out.stdout.strip() == "ok"
