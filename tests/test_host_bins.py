"""Host logic: the quantize kernel's bin tables (NF4 and FP4) and nearest-code
rule, checked exhaustively over every fp32 v in [-1, 1] by a small C++ program
built against the library's host tables (no GPU)."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_nf4_quantized_absmax_b200", "csrc")


@pytest.mark.timeout(600)
def test_bin_rule_matches_threshold_count_for_every_fp32(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    exe = str(tmp_path / "bins_check")
    subprocess.run([cxx, "-O2", "-std=c++17", "-pthread", f"-I{CSRC}",
                    os.path.join(ROOT, "tests", "host", "bins_check.cpp"), os.path.join(CSRC, "host_tables.cpp"),
                    "-o", exe], check=True)
    p = subprocess.run([exe], capture_output=True, text=True, timeout=560)
    assert p.returncode == 0, p.stdout + p.stderr
    lines = p.stdout.strip().splitlines()
    assert lines[-1] == "0 mismatches", p.stdout
    assert sum(1 for l in lines if l.endswith(", 0 mismatches")) == 2, p.stdout  # NF4 and FP4 tables
