"""Ragged-batch index mapping (csrc/segments.h), checked on the host.

The kernels of the one-launch ragged batch map work items, rows and groups
through the inline functions of segments.h; tests/segments_check.cpp calls
the same functions on random batches and checks coverage and containment
(every causal (row, key tile) scored by exactly one work item, no item
mixing sequences, every Refine member scored once with its own group, the
groups partitioning the tokens).  The PIVOT abstract groups consecutive
queries of one sequence; the batching itself is not on the pages.
"""
import shutil
import subprocess
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_segment_mapping_covers_every_pair_once(tmp_path):
    exe = tmp_path / "segments_check"
    subprocess.run(["g++", "-std=c++17", "-O2", "-Wall", "-Werror",
                    "-I", str(ROOT / "top_token_selection_b200" / "csrc"),
                    str(ROOT / "tests" / "segments_check.cpp"), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stdout + res.stderr
    assert res.stdout.startswith("ok ")
