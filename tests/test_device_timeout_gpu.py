"""Device-side failure detection, tested without a GPU fault: a bounded wait in
the attention kernel that runs out makes the kernel record a timeout in the
device error word and wind down (every load it issued lands, the tensor-core
work drains, tensor memory is freed) instead of hanging; the host reads the
status, and the same context and plan go on to compute correct results.

It runs the test-only build liblcsa_stalltest.so (-DLCSA_TEST_STALL: waits
give up after 100 ms; lcsa_test_arm_stall makes the next attention launch
give up on purpose) in a child process, so the product library is never
loaded beside it. Ways to give up, each on 128-token blocks and on the
paired 64-token path:
  site 1: the TMA producer gives up right after issuing its first work item's
          loads, while they are still in flight;
  site 2: a softmax warp waits on a barrier nothing arrives on, until the
          limit (the waits held up behind it run out at the same time, and
          the first to give up records its site);
  site 3 (with at least as many 64-token pairs as SMs, so the last pairs are
          cut into parts): one part of the first cut pair never flags its
          partial result, and the part that merges waits for it until the
          limit (site 27, the merge's wait).
Then lcsa_check_device_error must return LCSA_ERR_DEVICE_TIMEOUT, and the next
call on the same plan must match the fp64 oracle. The same holds for the
allocation-free entry point and its status call.
"""
import os
import subprocess
import sys

import pytest

from block_sparse_video_lcsa_b200 import build as lcsa_build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import numpy as np
import torch
import block_sparse_video_lcsa_b200 as L
import oracle
from block_sparse_video_lcsa_b200 import build, synth
from lcsa_harness import OUT_MAX_ABS, OUT_MEAN_ABS, block_rows_to_raster, torch_inputs

L.LIB_PATH = build.STALL_LIB      # the test-only build, in this process only
lib = L.lib()
arm = lib.lcsa_test_arm_stall
arm.restype = None

T = synth.WORKLOADS["tiny"]
CASES = {{
    "blocks128": T.replace(heads=3, q_frames=1, kv_frames=3, grid_h=24, grid_w=48, block_w=16, local_range=3,
                           topk=5, kv_frame_offset=2, field=True, unit_gain=False),
    "blocks64": T.replace(heads=2, q_frames=2, kv_frames=4, grid_h=32, grid_w=40, local_range=5, topk=9,
                          field=True, unit_gain=False, seed=3),
    # 160 pairs: the last are cut into parts and merged
    "blocks64_cut_pairs": T.replace(heads=8, q_frames=2, kv_frames=4, grid_h=32, grid_w=40, local_range=5, topk=9,
                                    field=True, unit_gain=False, seed=27),
}}

def err_vs_oracle(wl, inp, out):
    og = oracle.Geometry.from_workload(wl)
    _, _, _, ref, _ = oracle.run(og, inp)
    got = synth.bf16_bits_to_f64(out.view(torch.int16).cpu().numpy().view(np.uint16))
    D = og.head_dim
    e = np.concatenate([np.abs(got[b, tok, h * D:(h + 1) * D] - ref[n, i])
                        for b, tok, h, n, i in block_rows_to_raster(og, np.arange(og.rows), ref)])
    return float(e.max()), float(e.mean())

stream = torch.cuda.current_stream().cuda_stream
for name, wl in CASES.items():
    inp = synth.make_inputs(wl)
    q, k, v, gq, gk = torch_inputs(inp)
    plan = L.lcsa_plan_create(L.config_from_workload(wl), 0)
    for site in ((1, 2, 3) if "cut" in name else (1, 2)):
        out = torch.full_like(q, float("nan"))
        arm(site)
        plan.lcsa_forward(q, k, v, gq, gk, out)
        st = lib.lcsa_check_device_error(plan.handle, stream)
        msg = lib.lcsa_last_error_message().decode()
        assert st == L.LCSA_ERR_DEVICE_TIMEOUT, (name, site, st, msg)
        # site 1 records at once; at site 2 the waits held up behind the
        # stalled warp (the P.V issuer's, a partner's exchange) run out at the
        # same limit, and whichever is first records its own site
        assert {{1: "site 91", 2: "site ", 3: "site 27"}}[site] in msg, msg
        # the next call on the same plan and context is correct
        out = torch.full_like(q, float("nan"))
        plan.lcsa_forward(q, k, v, gq, gk, out)
        plan.lcsa_check_device_error()
        mx, mean = err_vs_oracle(wl, inp, out)
        assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, (name, site, mx, mean)
        print("%s site %d: timeout reported (%s); next call max %.3g mean %.3g" % (name, site, msg, mx, mean))
    plan.destroy()
    # the allocation-free entry point: its error word reports the timeout too
    cfg = L.config_from_workload(wl)
    out = torch.full_like(q, float("nan"))
    arm(1)
    assert L.lcsa_forward_noalloc(cfg, q, k, v, gq, gk, out) == L.LCSA_OK
    assert L.lcsa_noalloc_check_device_error() == L.LCSA_ERR_DEVICE_TIMEOUT
    assert L.lcsa_noalloc_check_device_error() == L.LCSA_OK        # read and cleared
    assert L.lcsa_forward_noalloc(cfg, q, k, v, gq, gk, out) == L.LCSA_OK
    assert L.lcsa_noalloc_check_device_error() == L.LCSA_OK
    mx, mean = err_vs_oracle(wl, inp, out)
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, (name, "noalloc", mx, mean)
    print("%s noalloc: timeout reported; next call max %.3g mean %.3g" % (name, mx, mean))
print("device-timeout test ok")
"""


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    lib = lcsa_build.build(stalltest=True)
    assert os.path.exists(lib)
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    sys.stdout.write(r.stdout)
    assert r.returncode == 0 and "device-timeout test ok" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
