"""The query-block pair enumeration of the 64-token path (which blocks may
pair, every block in exactly one pair) and the rule that picks the pairs to
cut, checked on the host: tests/pair_enumeration_check.cu includes the
library's internal header, is compiled here with nvcc (host code only) and
run. No GPU."""
import os
import subprocess

from block_sparse_video_lcsa_b200 import build as lcsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_every_query_block_is_in_exactly_one_pair(tmp_path):
    src = os.path.join(ROOT, "tests", "pair_enumeration_check.cu")
    exe = str(tmp_path / "pair_enumeration_check")
    inc = ["-I", os.path.join(ROOT, "include"), "-I", os.path.join(ROOT, "block_sparse_video_lcsa_b200", "csrc")]
    r = subprocess.run([lcsa_build.NVCC, "-std=c++17", "-O1"] + inc + [src, "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout[-2000:] + r.stderr[-2000:]
