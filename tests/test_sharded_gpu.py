"""Head-sharded layers through the C ABI: each emulated rank holds a slice of
the heads, the per-token sums of squares of all ranks are added (the sum the
ranks' all-reduce produces), and every rank's output and selection, put back
together, must match the fp64 oracle of the unsharded layer. The ranks run one
after another on one GPU: none of their kernels waits for another rank."""
import numpy as np
import pytest

import block_sparse_video_lcsa_b200 as L
import oracle
from block_sparse_video_lcsa_b200 import synth
from block_sparse_video_lcsa_b200.sharded import forward_heads_sharded, head_slices, sumsq_buffer

from lcsa_harness import (OUT_MAX_ABS, OUT_MEAN_ABS, GpuResult, check_output, check_selection, oracle_geometry,
                          sample_rows, torch_inputs)

pytestmark = pytest.mark.gpu

_T = synth.WORKLOADS["tiny"]
CASES = {
    # name: (workload, ranks)
    "tiny_2": (_T, 2),
    "stream_small_2": (_T.replace(heads=3, q_frames=1, kv_frames=3, grid_h=24, grid_w=48, block_w=16, local_range=3,
                                  topk=5, kv_frame_offset=2, field=True, unit_gain=False), 2),
    "blocks64_batch2_3": (_T.replace(batch=2, heads=5, q_frames=2, kv_frames=4, grid_h=32, grid_w=40, local_range=5,
                                     topk=9, field=True, unit_gain=False, seed=1), 3),
}


def run_sharded(wl, inp, ranks):
    """Emulated ranks on one GPU: returns the assembled GpuResult and the summed sums of squares."""
    import torch
    q, k, v, gq, gk = torch_inputs(inp)
    D = wl.head_dim
    plans, parts = [], []
    try:
        for h0, h1 in head_slices(wl.heads, ranks):
            cfg = L.config_from_workload(wl, heads=h1 - h0, heads_total=wl.heads)
            plan = L.lcsa_plan_create(cfg, 0)
            plans.append(plan)
            sl = slice(h0 * D, h1 * D)
            parts.append(tuple(t[..., sl].contiguous() for t in (q, k, v, gq, gk)) + (h0, h1))
        # step 1 on every rank, then the all-reduce (a sum over the ranks)
        ss = [sumsq_buffer(p, q.device) for p in plans]
        for p, part, s in zip(plans, parts, ss):
            p.lcsa_sumsq(part[0], part[1], s)
        total = torch.stack(ss).sum(0)
        outs = []
        for p, part in zip(plans, parts):
            o = torch.empty_like(part[0])
            p.lcsa_forward_sharded(*part[:5], total, o)
            outs.append(o)
        for p in plans:
            p.lcsa_check_device_error()
        torch.cuda.synchronize()
        out = torch.cat(outs, dim=-1).view(torch.int16).cpu().numpy().view(np.uint16)
        # CSR rows of the full layer: (b, h, qb) with h = the rank's h0 + its own head index
        sels = [p.lcsa_get_selection() for p in plans]
        nQB = plans[0].geometry.q_blocks
        rows, nnz = [], 0
        for b in range(wl.batch):
            for (rp, ci), (h0, h1) in zip(sels, [pt[5:] for pt in parts]):
                for hl in range(h1 - h0):
                    for qb in range(nQB):
                        r = (b * (h1 - h0) + hl) * nQB + qb
                        rows.append(ci[rp[r]:rp[r + 1]])
        row_ptr = np.zeros(len(rows) + 1, dtype=np.int32)
        np.cumsum([r.size for r in rows], out=row_ptr[1:])
        col_idx = np.concatenate(rows).astype(np.int32)
        return GpuResult(out, row_ptr, col_idx, None, None, None, None, None), total.cpu().numpy()
    finally:
        for p in plans:
            p.destroy()


@pytest.mark.parametrize("name", list(CASES))
def test_sharded_layer_matches_unsharded_oracle(name):
    wl, ranks = CASES[name]
    inp = synth.make_inputs(wl)
    og = oracle_geometry(wl)
    gpu, ss = run_sharded(wl, inp, ranks)
    # the summed per-token sums of squares are those of the whole layer
    xq = synth.bf16_bits_to_f64(inp.q).reshape(-1, og.C)
    xk = synth.bf16_bits_to_f64(inp.k).reshape(-1, og.C)
    want = np.concatenate([(xq * xq).sum(1), (xk * xk).sum(1)])
    np.testing.assert_allclose(ss, want, rtol=2e-6, atol=1e-6)
    pq = oracle.pool(og, inp.q, inp.gamma_q, True)
    pk = oracle.pool(og, inp.k, inp.gamma_k, False)
    sel = oracle.select(og, pq, pk, want_scores=True)
    gsel, _, _ = check_selection(og, sel, gpu)
    rows = sample_rows(og, 64)
    out, _ = oracle.attention(og, inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k, gsel, rows)
    mx, mean = check_output(og, gpu, rows, out)
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, (mx, mean)


def test_one_rank_helper_equals_plain_forward():
    """heads_total == heads: forward_heads_sharded (no process group) is the plain call, bit for bit."""
    import torch
    wl = CASES["stream_small_2"][0]
    inp = synth.make_inputs(wl)
    q, k, v, gq, gk = torch_inputs(inp)
    plan = L.lcsa_plan_create(L.config_from_workload(wl), 0)
    try:
        a, b = torch.empty_like(q), torch.empty_like(q)
        plan.lcsa_forward(q, k, v, gq, gk, a)
        forward_heads_sharded(plan, q, k, v, gq, gk, b)
        plan.lcsa_check_device_error()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    finally:
        plan.destroy()


def test_sharded_plan_rejects_the_plain_call():
    import torch
    wl = CASES["tiny_2"][0]
    inp = synth.make_inputs(wl)
    q, k, v, gq, gk = torch_inputs(inp)
    D = wl.head_dim
    plan = L.lcsa_plan_create(L.config_from_workload(wl, heads=1, heads_total=2), 0)
    try:
        part = [t[..., :D].contiguous() for t in (q, k, v, gq, gk)]
        with pytest.raises(L.LcsaError) as e:
            plan.lcsa_forward(*part, torch.empty_like(part[0]))
        assert e.value.status == L.LCSA_ERR_INVALID_ARG
    finally:
        plan.destroy()
    # head scope needs no exchange: the plain call serves a sharded plan, and
    # its output equals the same heads of the unsharded head-scope layer
    full = L.lcsa_plan_create(L.config_from_workload(wl, norm_scope=L.LCSA_NORM_HEAD), 0)
    half = L.lcsa_plan_create(L.config_from_workload(wl, heads=1, heads_total=2, norm_scope=L.LCSA_NORM_HEAD), 0)
    try:
        a = torch.empty_like(q)
        full.lcsa_forward(q, k, v, gq, gk, a)
        part = [t[..., D:].contiguous() for t in (q, k, v, gq, gk)]
        b = torch.empty_like(part[0])
        half.lcsa_forward(*part, b)
        with pytest.raises(L.LcsaError):
            half.lcsa_forward_sharded(*part, sumsq_buffer(half, q.device), b)
        torch.cuda.synchronize()
        assert torch.equal(a[..., D:].contiguous().view(torch.int16), b.view(torch.int16))
    finally:
        full.destroy()
        half.destroy()
