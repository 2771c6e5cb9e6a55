"""include/msda.h is plain C: a C99 program (tests/c/abi_check.c) compiled
with gcc -std=c99 -Wall -Werror links libmsda.so and runs the host-side
queries and argument checks of the ABI (no GPU needed)."""
import os
import subprocess

import pytest

from scale_deformable_attention_msdeformattn_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_header_is_c99_and_abi_is_callable_from_c(tmp_path):
    lib = build.build()
    exe = str(tmp_path / "abi_check")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_check.c"),
           "-L", os.path.dirname(lib), "-l:" + os.path.basename(lib),
           "-Wl,-rpath," + os.path.dirname(lib), "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    res = subprocess.run([exe], capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "0 failure(s)" in res.stdout
