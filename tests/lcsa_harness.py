"""Shared helpers of the GPU parity tests: run the CUDA library through its C
ABI and compare with the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import dataclasses

import numpy as np

import block_sparse_video_lcsa_b200 as L
import oracle
from block_sparse_video_lcsa_b200 import synth

# Tolerances of the bf16 output against the fp64 oracle, and the near-tie
# threshold below which two block scores count as tied.
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
TIE_GAP = 1e-4


def torch_inputs(inp: synth.Inputs, device="cuda:0"):
    import torch

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(device)

    return (bf(inp.q), bf(inp.k), bf(inp.v), torch.from_numpy(inp.gamma_q).to(device),
            torch.from_numpy(inp.gamma_k).to(device))


@dataclasses.dataclass
class GpuResult:
    out: np.ndarray        # uint16 bf16 bits [B, Lq, C]
    row_ptr: np.ndarray
    col_idx: np.ndarray
    qhat: np.ndarray
    khat: np.ndarray
    pooled_q: np.ndarray
    pooled_k: np.ndarray
    geometry: object


def run_gpu(wl: synth.Workload, inp: synth.Inputs, calls: int = 1, **cfg_over) -> GpuResult:
    import torch
    cfg = L.config_from_workload(wl, **cfg_over)
    plan = L.lcsa_plan_create(cfg, 0)
    try:
        q, k, v, gq, gk = torch_inputs(inp)
        out = torch.empty_like(q)
        for _ in range(calls):
            plan.lcsa_forward(q, k, v, gq, gk, out)
        plan.lcsa_check_device_error()
        torch.cuda.synchronize()
        rp, ci = plan.lcsa_get_selection()
        qh, kh, pq, pk = plan.lcsa_get_intermediates()
        o = out.view(torch.int16).cpu().numpy().view(np.uint16)
        return GpuResult(o, rp, ci, qh, kh, pq, pk, plan.geometry)
    finally:
        plan.destroy()


def oracle_geometry(wl, **over):
    return oracle.Geometry.from_workload(wl, **over)


def check_selection(og, sel: oracle.Selection, gpu: GpuResult):
    """GPU CSR == oracle CSR bit for bit, except rows whose k-th / (k+1)-th
    oracle scores are closer than TIE_GAP; those rows must still hold a valid
    choice (right length, ascending, admissible, each kept score within TIE_GAP
    of the k-th best). Returns the GPU selection as an oracle.Selection."""
    rows = og.rows
    rp = gpu.row_ptr.astype(np.int64)
    assert rp.size == rows + 1
    want_len = sel.row_len.astype(np.int64)
    np.testing.assert_array_equal(np.diff(rp), want_len)
    cap = sel.cols.shape[1]
    gcols = np.full((rows, cap), -1, dtype=np.int32)
    near = np.flatnonzero(sel.gap < TIE_GAP)
    mism = []
    for r in range(rows):
        g = gpu.col_idx[rp[r]:rp[r + 1]]
        gcols[r, : g.size] = g
        if not np.array_equal(g, sel.row(r)):
            mism.append(r)
    bad = sorted(set(mism) - set(near.tolist()))
    assert not bad, "CSR differs on %d rows that are not near-ties, e.g. %s" % (len(bad), bad[:5])
    if mism:
        assert sel.scores is not None
        for r in mism:
            g = gcols[r, : want_len[r]]
            assert np.all(np.diff(g) > 0)
            sc = sel.scores[r]
            assert np.all(np.isfinite(sc[g])), "non-admissible block kept"
            kth = np.sort(sc[np.isfinite(sc)])[::-1][want_len[r] - 1]
            assert np.all(sc[g] >= kth - TIE_GAP)
    return oracle.Selection(want_len.astype(np.int32), gcols, sel.gap, sel.scores), len(mism), near.size


def block_rows_to_raster(og, rows, blocks_out):
    """Scatter oracle outputs [n, nb, d] of rows into raster [(b, token), h, d] keys."""
    nWb = og.grid_w // og.block_w
    bpf = og.blocks_per_frame
    res = []
    for n, row in enumerate(rows):
        bh, qb = divmod(int(row), og.nQB)
        b, h = divmod(bh, og.heads)
        tb, rem = divmod(qb, bpf)
        hb, wb = divmod(rem, nWb)
        i = 0
        for tt in range(og.block_t):
            for yy in range(og.block_h):
                for xx in range(og.block_w):
                    t, y, x = tb * og.block_t + tt, hb * og.block_h + yy, wb * og.block_w + xx
                    tok = (t * og.grid_h + y) * og.grid_w + x
                    res.append((b, tok, h, n, i))
                    i += 1
    return res


def check_output(og, gpu: GpuResult, rows, ref):
    """GPU bf16 output vs the oracle's fp64 output of `rows` ([n, nb, d])."""
    out = synth.bf16_bits_to_f64(gpu.out)
    D = og.head_dim
    errs = []
    for b, tok, h, n, i in block_rows_to_raster(og, rows, ref):
        errs.append(np.abs(out[b, tok, h * D:(h + 1) * D] - ref[n, i]))
    e = np.concatenate(errs)
    assert np.all(np.isfinite(out))
    return float(e.max()), float(e.mean())


def sample_rows(og, count, seed=0):
    rows = og.rows
    if rows <= count:
        return np.arange(rows, dtype=np.int64)
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(rows, size=count - 4, replace=False).tolist())
    pick |= {0, og.nQB - 1, rows - og.nQB, rows - 1}      # corners of the first and last head
    return np.array(sorted(pick), dtype=np.int64)
