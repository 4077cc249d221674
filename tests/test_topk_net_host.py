"""The register Top-K level merge of the CUDA path, compiled for the host, against a plain
sort of all candidates of a level (RAM-Net project page, exactness paragraph after the five
views: the level's K best are among the extensions of the previous level's K best).

Random kept lists and digit codes, including repeated digit scores (the index tie-break),
for N in {8, 16, 32} and up to 16 digit values.  Needs nvcc, no GPU.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "native", "topk_net_check.cu")


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_register_topk_merge_matches_sort(tmp_path):
    exe = str(tmp_path / "topk_net_check")
    subprocess.run(["nvcc", "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a", "-o", exe, SRC],
                   check=True, capture_output=True, timeout=300)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=300).stdout
    checked, bad = int(out.split()[1]), int(out.split()[3])
    assert checked > 100000 and bad == 0, out
