"""lcsa_forward_host, the call from host buffers: the inputs go up in the
order the kernels need them (q and k on the call's stream, v on the plan's
copy stream while the prologue and the selection run), and with one batch
element and two or more heads the attention runs as two launches over the
two halves of the heads, the first half's output channels coming back while
the second half computes. Rows are independent, so the result must equal the
device-buffer call on the same plan bit for bit, on two calls in a row with
different inputs; one case is also compared with the fp64 oracle.
"""
import numpy as np
import pytest

import block_sparse_video_lcsa_b200 as L
import oracle
from block_sparse_video_lcsa_b200 import synth

from lcsa_harness import OUT_MAX_ABS, OUT_MEAN_ABS, block_rows_to_raster, torch_inputs

pytestmark = pytest.mark.gpu

_T = synth.WORKLOADS["tiny"]
CASES = {
    # split into two attention launches (3 heads: 1 + 2)
    "blocks128_split": _T.replace(heads=3, q_frames=1, kv_frames=3, grid_h=24, grid_w=48, block_w=16,
                                  local_range=3, topk=5, kv_frame_offset=2, field=True, unit_gain=False),
    # paired 64-token query tiles, split by pairs
    "blocks64_split": _T.replace(heads=4, q_frames=2, kv_frames=4, grid_h=32, grid_w=40, local_range=5, topk=9,
                                 field=True, unit_gain=False, seed=3),
    # one head: a single launch
    "one_head": _T.replace(heads=1, field=True, unit_gain=False, seed=5),
    # two batch elements: a single launch
    "batch2": _T.replace(batch=2, heads=2, topk=3, field=True, unit_gain=False, seed=6),
    "d64_split": _T.replace(head_dim=64, heads=4, q_frames=1, kv_frames=3, grid_h=24, grid_w=48, block_w=16,
                            local_range=3, topk=5, field=True, unit_gain=False, seed=7),
    # 160 query-block pairs, at least as many as the SMs: the last pairs are cut and merged
    "cut_pairs": _T.replace(heads=8, q_frames=2, kv_frames=4, grid_h=32, grid_w=40, local_range=5, topk=9,
                            field=True, unit_gain=False, seed=22),
}


@pytest.mark.parametrize("name", list(CASES))
def test_host_buffers_give_the_device_call_bit_for_bit(name):
    import torch
    wl = CASES[name]
    plan = L.lcsa_plan_create(L.config_from_workload(wl, host_io=1), 0)
    try:
        for seed in (0, 1):
            inp = synth.make_inputs(wl.replace(seed=wl.seed + 10 * seed))
            dev = torch_inputs(inp)
            want = torch.empty_like(dev[0])
            plan.lcsa_forward(*dev, want)
            plan.lcsa_check_device_error()
            host = [t.cpu().pin_memory() for t in dev]
            got = torch.full_like(host[0], float("nan")).pin_memory()
            plan.lcsa_forward_host(*host, got)
            a = got.view(torch.int16).numpy()
            b = want.view(torch.int16).cpu().numpy()
            diff = int(np.count_nonzero(a != b))
            assert diff == 0, "call %d: %d output elements differ from the device-buffer call" % (seed, diff)
        if name == "blocks64_split":
            og = oracle.Geometry.from_workload(wl.replace(seed=wl.seed + 10))
            _, _, _, ref, _ = oracle.run(og, inp)
            out = synth.bf16_bits_to_f64(a.view(np.uint16))
            D = og.head_dim
            err = np.concatenate([np.abs(out[bb, tok, h * D:(h + 1) * D] - ref[n, i])
                                  for bb, tok, h, n, i in block_rows_to_raster(og, np.arange(og.rows), ref)])
            assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (err.max(), err.mean())
    finally:
        plan.destroy()
