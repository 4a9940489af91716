"""bench.py host logic on CPU: the launch count it claims per call and the
recorded DRAM traffic it attaches to the roofline (only for the workload and
kernel source the capture was taken on)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_sparse_video_lcsa_b200 import synth  # noqa: E402

K3_FILES = ["k3_attention_tc.cu", "lcsa_internal.h"]


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_launch_count_per_call(name):
    wl = synth.WORKLOADS[name]
    nb = wl.block_t * wl.block_h * wl.block_w
    # K1, K2, K3; 64-token blocks add the pair-union kernel between K2 and K3
    assert bench._launches_per_call(wl) == (4 if nb == 64 else 3)


def _records():
    out = []
    with open(os.path.join(ROOT, "profiles", "dram_traffic.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                fields = dict(kv.split("=", 1) for kv in line.split()[1:])
                out.append((line.split()[0], fields["src"], fields["workload"], float(fields["dram_bytes_per_launch"])))
    return out


def test_recorded_traffic_is_keyed_by_workload_and_source():
    recs = _records()
    assert recs, "no traffic record"
    src = bench._kernel_source_hash(K3_FILES)
    for tag, h, wl, nbytes in recs:
        assert wl in synth.WORKLOADS, wl
        got = bench._profiled_traffic(tag, K3_FILES, wl)
        assert got == (nbytes if h == src else None)
    recorded = {wl for _, _, wl, _ in recs}
    for wl in synth.WORKLOADS:
        if wl not in recorded:
            assert bench._profiled_traffic("k3", K3_FILES, wl) is None


def test_recorded_traffic_is_dropped_once_the_source_changes(monkeypatch):
    monkeypatch.setattr(bench, "_kernel_source_hash", lambda files: "0" * 16)
    for wl in synth.WORKLOADS:
        assert bench._profiled_traffic("k3", K3_FILES, wl) is None


def test_source_hash_ignores_comments_but_not_code():
    a = 'int f(int x) {  // twice\n  return 2 * x; /* doubled */ }\nconst char* s = "a // b";\n'
    b = '/* header */\nint f(int x) {\n\n  return 2 * x;\n}\nconst char* s = "a // b";  // string kept\n'
    c = 'int f(int x) { return 3 * x; }\nconst char* s = "a // b";\n'
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    assert '"a // b"' in bench._code_only(a)


def test_reference_arm_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints
    one JSON line with the contract's keys, on the same workload keys as the
    CUDA arm's line."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "dtype", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    wl = synth.WORKLOADS[d["config"]["workload"]]
    assert d["config"]["q_tokens"] == wl.q_tokens and d["config"]["kv_tokens"] == wl.kv_tokens
    assert d["config"]["kept_blocks"] == 43200  # 720 rows x 60 blocks on the default workload


def test_spread_of_call_times():
    d = bench._spread([5.0, 1.0, 3.0, 2.0, 4.0])
    assert d == {"p10": 1.4, "median": 3.0, "p90": 4.6}
    assert bench._spread([0.41]) == {"p10": 0.41, "median": 0.41, "p90": 0.41}
