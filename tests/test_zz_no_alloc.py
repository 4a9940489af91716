"""lcsa_forward_noalloc, the entry point for callers that may not allocate
device memory while they run (for example a real-time video pipeline or a
plugin whose device memory is reserved at start-up: a cudaMalloc there would
synchronise the device and stall the other streams, or fail outright).

It runs the plan path's kernels on the same inputs, so its output must equal
the plan path's bit for bit, on two calls in a row with different inputs (the
shared static workspace keeps the previous call's contents); one case is also
compared with the fp64 oracle at the parity tolerance, and the static
workspace's error word must read clean afterwards. This file is collected
last on purpose.
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
    "tiny": _T,
    "stream_small": _T.replace(heads=3, q_frames=1, kv_frames=3, grid_h=24, grid_w=48, block_w=16, local_range=3,
                               topk=5, kv_frame_offset=2, field=True, unit_gain=False),
    "blocks64_d64": _T.replace(head_dim=64, heads=4, q_frames=2, kv_frames=4, grid_h=32, grid_w=40, local_range=5,
                               topk=9, field=True, unit_gain=False, seed=13),
    # 160 query-block pairs, at least as many as the SMs: the last pairs are cut and merged
    "cut_pairs": _T.replace(heads=8, q_frames=2, kv_frames=4, grid_h=32, grid_w=40, local_range=5, topk=9,
                            field=True, unit_gain=False, seed=22),
}


def _plan_output(wl, inp):
    import torch
    plan = L.lcsa_plan_create(L.config_from_workload(wl), 0)
    try:
        q, k, v, gq, gk = torch_inputs(inp)
        out = torch.empty_like(q)
        plan.lcsa_forward(q, k, v, gq, gk, out)
        plan.lcsa_check_device_error()
        return out.view(torch.int16).cpu().numpy()
    finally:
        plan.destroy()


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_the_plan_path_on_two_calls_in_a_row(name):
    import torch
    wl = CASES[name]
    loads = [synth.make_inputs(wl.replace(seed=s)) for s in (0, 1)]
    want = [_plan_output(wl, inp) for inp in loads]
    cfg = L.config_from_workload(wl)
    tensors = [torch_inputs(inp) for inp in loads]
    outs = [torch.full_like(t[0], float("nan")) for t in tensors]
    for (q, k, v, gq, gk), out in zip(tensors, outs):          # back to back on one stream
        assert L.lcsa_forward_noalloc(cfg, q, k, v, gq, gk, out) == L.LCSA_OK
    assert L.lcsa_noalloc_check_device_error() == L.LCSA_OK
    for call, (out, ref) in enumerate(zip(outs, want)):
        got = out.view(torch.int16).cpu().numpy()
        diff = int(np.count_nonzero(got != ref))
        assert diff == 0, "call %d: %d output elements differ from the plan path" % (call, diff)
    # the second call against the fp64 oracle as well (parity tolerance)
    og = oracle.Geometry.from_workload(wl)
    _, _, _, ref, _ = oracle.run(og, loads[1])
    got = synth.bf16_bits_to_f64(outs[1].view(torch.int16).cpu().numpy().view(np.uint16))
    D = og.head_dim
    err = np.concatenate([np.abs(got[b, tok, h * D:(h + 1) * D] - ref[n, i])
                          for b, tok, h, n, i in block_rows_to_raster(og, np.arange(og.rows), ref)])
    assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (err.max(), err.mean())


def test_noalloc_rejects_problems_larger_than_its_workspace():
    import torch
    cfg = L.config_from_workload(synth.WORKLOADS["stream_768x1280"])
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda:0")
    g = torch.ones(16, dtype=torch.float32, device="cuda:0")
    assert L.lcsa_forward_noalloc(cfg, x, x, x, g, g, x) == L.LCSA_ERR_UNSUPPORTED
    assert L.lcsa_noalloc_check_device_error() == L.LCSA_OK
