"""Host-side test (no GPU) of the per-device set-up bookkeeping the decode
launcher uses for kernel attributes (csrc/kvq_devonce.h): set up once per
device ordinal, each device on its own, failures retried, safe under
concurrent host threads.  The header is plain C++; it is compiled here with
g++ into a small harness."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_once_per_device(tmp_path):
    exe = tmp_path / "devonce"
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread",
                    "-I", os.path.join(ROOT, "decode_attention_kvq_b200", "csrc"),
                    os.path.join(ROOT, "tests", "host", "devonce_harness.cpp"), "-o", str(exe)],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
