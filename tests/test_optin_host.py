"""The per-device shared-memory opt-in record of the library's launchers
(csrc/optin.h), compiled with the host C++ compiler and driven by a fake
setter: one attribute call per device and size, retries after a failure,
thread safety.  No GPU needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "native", "optin_table_test.cpp")
INC = os.path.join(ROOT, "block_sparse_attention_candidate_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_optin_table(tmp_path):
    exe = str(tmp_path / "optin_table_test")
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", INC, SRC, "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
