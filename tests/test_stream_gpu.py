"""Stream plans (lcsa_plan_create_stream / lcsa_stream_push /
lcsa_forward_stream) against the stateless fp64 oracle.

A sequence of frames is pushed chunk by chunk ("FlashVSR: From 17.2 FPS to
57.3 FPS at 768x1408", Rebuild sparse attention for Hopper: incremental pooled-K
caching; "FlashVSR Inference", Non-Negotiable Streaming Contract: KV window =
kv_ratio x query frames). After each chunk the output must equal the oracle's
stateless call on that window (query frames = the chunk, KV = the last
kv_frames frames, RoPE positions from the window's absolute first frame):
selection bit-exact outside near-ties, output within the parity tolerance.
"""
import numpy as np
import pytest

import oracle
from block_sparse_video_lcsa_b200 import synth
import block_sparse_video_lcsa_b200 as L

from lcsa_harness import OUT_MAX_ABS, OUT_MEAN_ABS, check_output, check_selection, oracle_geometry

pytestmark = pytest.mark.gpu

_T = synth.WORKLOADS["tiny"]
STREAMS = {
    # 128-token blocks, windowed selection
    "stream128": _T.replace(heads=3, q_frames=2, kv_frames=6, grid_h=24, grid_w=48, block_w=16, local_range=3,
                            topk=5, field=True, unit_gain=False, seed=8),
    # 64-token blocks (paired 128-row query tiles), an odd top-k (a half KV tile per row)
    "stream64": _T.replace(heads=2, q_frames=2, kv_frames=6, grid_h=32, grid_w=40, local_range=5, topk=7,
                           field=True, unit_gain=False, seed=9),
    # head_dim 64
    "stream128_d64": _T.replace(head_dim=64, heads=4, q_frames=2, kv_frames=6, grid_h=24, grid_w=48, block_w=16,
                                local_range=3, topk=5, field=True, unit_gain=False, seed=12),
    # 160 query-block pairs, at least as many as the SMs: the last pairs are cut and merged
    "stream64_cut_pairs": _T.replace(heads=8, q_frames=2, kv_frames=6, grid_h=32, grid_w=40, local_range=5, topk=7,
                                     field=True, unit_gain=False, seed=24),
}
TOTAL_FRAMES = 10   # 4 pushed to fill the window, then three chunks of 2


@pytest.mark.parametrize("name", list(STREAMS))
def test_stream_chunks_equal_stateless_windows(name):
    import torch
    wl = STREAMS[name]
    seq = synth.make_inputs(wl.replace(q_frames=TOTAL_FRAMES, kv_frames=TOTAL_FRAMES))
    plane = wl.grid_h * wl.grid_w
    frames = lambda a, f0, f1: np.ascontiguousarray(a[:, f0 * plane:f1 * plane, :])  # noqa: E731
    dev = torch.device("cuda:0")
    bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).to(dev)  # noqa: E731
    gq, gk = torch.from_numpy(seq.gamma_q).to(dev), torch.from_numpy(seq.gamma_k).to(dev)
    plan = L.lcsa_plan_create_stream(L.config_from_workload(wl), 0)
    try:
        first = wl.kv_frames - wl.q_frames
        plan.lcsa_stream_push(bf(frames(seq.k, 0, first)), bf(frames(seq.v, 0, first)), gk, first)
        for chunk, f0 in enumerate(range(first, TOTAL_FRAMES, wl.q_frames)):
            f1 = f0 + wl.q_frames
            out = torch.full((wl.batch, wl.q_frames * plane, wl.channels), float("nan"), dtype=torch.bfloat16,
                             device=dev)
            plan.lcsa_forward_stream(bf(frames(seq.q, f0, f1)), bf(frames(seq.k, f0, f1)),
                                     bf(frames(seq.v, f0, f1)), gq, gk, out)
            plan.lcsa_check_device_error()
            w0 = f1 - wl.kv_frames   # absolute first frame of the window
            win = synth.Inputs(q=frames(seq.q, f0, f1), k=frames(seq.k, w0, f1), v=frames(seq.v, w0, f1),
                               gamma_q=seq.gamma_q, gamma_k=seq.gamma_k)
            og = oracle_geometry(wl.replace(kv_frame_offset=w0))
            pq = oracle.pool(og, win.q, win.gamma_q, True)
            pk = oracle.pool(og, win.k, win.gamma_k, False)
            sel = oracle.select(og, pq, pk, want_scores=True)
            rp, ci = plan.lcsa_get_selection()

            class _G:  # the fields check_selection / check_output read
                pass
            gpu = _G()
            gpu.row_ptr, gpu.col_idx = rp, ci
            gpu.out = out.view(torch.int16).cpu().numpy().view(np.uint16)
            gsel, nmis, nnear = check_selection(og, sel, gpu)
            ref, _ = oracle.attention(og, win.q, win.k, win.v, win.gamma_q, win.gamma_k, gsel)
            mx, mean = check_output(og, gpu, np.arange(og.rows), ref)
            assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, (chunk, mx, mean)
    finally:
        plan.destroy()


def test_stream_plan_rejects_a_chunk_before_the_window_is_full():
    import torch
    wl = STREAMS["stream128"]
    plane = wl.grid_h * wl.grid_w
    dev = torch.device("cuda:0")
    x = torch.zeros((wl.batch, wl.q_frames * plane, wl.channels), dtype=torch.bfloat16, device=dev)
    g = torch.ones(wl.channels, dtype=torch.float32, device=dev)
    plan = L.lcsa_plan_create_stream(L.config_from_workload(wl), 0)
    try:
        with pytest.raises(L.LcsaError):
            plan.lcsa_forward_stream(x, x, x, g, g, torch.empty_like(x))
        kv = torch.zeros((wl.batch, wl.kv_frames * plane, wl.channels), dtype=torch.bfloat16, device=dev)
        with pytest.raises(L.LcsaError):
            plan.lcsa_forward(x, kv, kv, g, g, torch.empty_like(x))   # stream plans take the stream calls
    finally:
        plan.destroy()
