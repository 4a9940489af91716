"""Pins of the fp64 CPU oracle against facts it does not compute itself.

Each test checks a property that the mathematics or the pages fix (dense
limit, top-k definition, softmax identities, rotation invariants, closed forms)
so that a dropped term, a wrong sign or index or a swapped operand in the
oracle fails here. No GPU is used.
"""
import math

import numpy as np
import pytest

import oracle
from block_sparse_video_lcsa_b200 import synth


def tiny(**over):
    wl = synth.WORKLOADS["tiny"].replace(**over)
    return wl, oracle.Geometry.from_workload(wl)


def block_raster_tokens(g, blk):
    """Raster indices l = (t*H' + y)*W' + x of one block, written out here from
    the token-grid definition (independent of the oracle's own mapping)."""
    nWb = g.grid_w // g.block_w
    bpf = (g.grid_h // g.block_h) * nWb
    tb, rem = divmod(blk, bpf)
    hb, wb = divmod(rem, nWb)
    out = []
    for tt in range(g.block_t):
        for yy in range(g.block_h):
            for xx in range(g.block_w):
                t, y, x = tb * g.block_t + tt, hb * g.block_h + yy, wb * g.block_w + xx
                out.append((t * g.grid_h + y) * g.grid_w + x)
    return np.array(out, dtype=np.int64)


def dense_attention(qh, kh, vh, scale):
    """Textbook softmax(q k^T * scale) v in fp64."""
    s = (qh @ kh.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ vh


# --------------------------------------------------------------------------
# P1: with every block kept and no window, LCSA is dense attention.

@pytest.mark.parametrize("over", [
    dict(),                                                   # tiny: 2 frames of 16x16, 8x8 blocks
    dict(q_frames=1, kv_frames=3, kv_frame_offset=5),         # queries are the last frame of the window
    dict(grid_h=32, grid_w=32, q_frames=1, kv_frames=1),      # 4x4 block grid
    dict(block_w=16, grid_w=32, heads=3),                     # 128-token blocks, odd head count
])
def test_dense_limit_equals_softmax_attention(over):
    wl, g = tiny(local_range=0, **over)
    g.topk = g.nKB
    inp = synth.make_inputs(wl)
    pq, pk, sel, out, wsum = oracle.run(g, inp)
    assert np.all(sel.row_len == g.nKB)
    qt = oracle.norm_rope(g, inp.q, inp.gamma_q, True, np.arange(g.Lq))
    kt = oracle.norm_rope(g, inp.k, inp.gamma_k, False, np.arange(g.Lkv))
    v = synth.bf16_bits_to_f64(inp.v[0])
    D = g.head_dim
    for h in range(g.heads):
        ref = dense_attention(qt[:, h * D:(h + 1) * D], kt[:, h * D:(h + 1) * D], v[:, h * D:(h + 1) * D],
                              1.0 / math.sqrt(D))
        for qb in range(g.nQB):
            row = h * g.nQB + qb
            toks = block_raster_tokens(g, qb)
            np.testing.assert_allclose(out[row], ref[toks], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# P2: selection is the top-k of the admissible set with lower-index ties.

def _admissible_bruteforce(g, qb, kb):
    if g.local_range <= 0:
        return True
    r = (g.local_range - 1) // 2
    nWb = g.grid_w // g.block_w
    bpf = (g.grid_h // g.block_h) * nWb
    (qh, qw), (kh, kw) = divmod(qb % bpf, nWb), divmod(kb % bpf, nWb)
    return abs(qh - kh) <= r and abs(qw - kw) <= r


@pytest.mark.parametrize("lr,k,frames", [(3, 4, 2), (3, 1, 1), (3, 20, 3), (1, 2, 3), (5, 7, 2), (0, 5, 2)])
def test_topk_is_the_defined_selection_with_ties(lr, k, frames):
    # 4x4 block grid; integer-valued pooled vectors produce many exact ties
    g = oracle.Geometry(batch=2, heads=2, head_dim=4, q_frames=frames, kv_frames=frames, grid_h=32, grid_w=32,
                        block_t=1, block_h=8, block_w=8, local_range=lr, topk=k)
    rng = np.random.default_rng(lr * 100 + k)
    pq = rng.integers(-2, 3, size=(g.batch, g.heads, g.nQB, g.head_dim)).astype(np.float64)
    pk = rng.integers(-2, 3, size=(g.batch, g.heads, g.nKB, g.head_dim)).astype(np.float64)
    sel = oracle.select(g, pq, pk, want_scores=True)
    for b in range(g.batch):
        for h in range(g.heads):
            for qb in range(g.nQB):
                row = (b * g.heads + h) * g.nQB + qb
                adm = [kb for kb in range(g.nKB) if _admissible_bruteforce(g, qb, kb)]
                score = {kb: float(pq[b, h, qb] @ pk[b, h, kb]) for kb in adm}
                chosen = list(sel.row(row))
                assert len(chosen) == min(k, len(adm))
                assert chosen == sorted(set(chosen))
                assert set(chosen) <= set(adm)
                rest = [kb for kb in adm if kb not in chosen]
                for s in chosen:
                    for u in rest:
                        assert score[s] > score[u] or (score[s] == score[u] and s < u)
                ordered = sorted(score.values(), reverse=True)
                if len(chosen) < len(adm):
                    assert sel.gap[row] == ordered[len(chosen) - 1] - ordered[len(chosen)]
                else:
                    assert sel.gap[row] == np.inf
                for kb in range(g.nKB):
                    if kb in score:
                        assert sel.scores[row, kb] == score[kb]
                    else:
                        assert sel.scores[row, kb] == -np.inf


def test_window_sizes_closed_form():
    g = oracle.Geometry(batch=1, heads=1, head_dim=4, q_frames=2, kv_frames=3, grid_h=48, grid_w=40, block_t=1,
                        block_h=8, block_w=8, local_range=5, topk=1)
    nHb, nWb, r = 6, 5, 2
    sizes = oracle.window_sizes(g)
    for qb in range(g.nQB):
        hb, wb = divmod(qb % (nHb * nWb), nWb)
        nh = min(hb + r, nHb - 1) - max(hb - r, 0) + 1
        nw = min(wb + r, nWb - 1) - max(wb - r, 0) + 1
        assert sizes[qb] == g.kv_frames * nh * nw


def test_row_length_is_budget_clipped_to_window():
    wl, g = tiny(grid_h=48, grid_w=48, q_frames=1, kv_frames=2, local_range=3, topk=10)
    inp = synth.make_inputs(wl)
    pq = oracle.pool(g, inp.q, inp.gamma_q, True)
    pk = oracle.pool(g, inp.k, inp.gamma_k, False)
    sel = oracle.select(g, pq, pk)
    sizes = oracle.window_sizes(g)
    for row in range(g.rows):
        assert sel.row_len[row] == min(10, sizes[row % g.nQB])
        assert np.all(np.diff(sel.row(row)) > 0)


# --------------------------------------------------------------------------
# P3: softmax identities.

def test_constant_values_give_constant_output():
    wl, g = tiny()
    inp = synth.make_inputs(wl)
    inp.v[:] = synth.to_bf16_bits(np.full(inp.v.shape, 1.375))
    _, _, _, out, wsum = oracle.run(g, inp)
    np.testing.assert_allclose(out, 1.375, rtol=0, atol=1e-12)
    np.testing.assert_allclose(wsum, 1.0, rtol=0, atol=1e-12)


def test_zero_queries_average_the_selected_values():
    wl, g = tiny(grid_h=32, grid_w=32, local_range=3)
    inp = synth.make_inputs(wl)
    inp.q[:] = 0
    _, _, sel, out, _ = oracle.run(g, inp)
    v = synth.bf16_bits_to_f64(inp.v[0])
    D = g.head_dim
    for row in range(g.rows):
        h, qb = divmod(row, g.nQB)
        toks = np.concatenate([block_raster_tokens(g, kb) for kb in sel.row(row)])
        mean = v[toks, h * D:(h + 1) * D].mean(axis=0)
        np.testing.assert_allclose(out[row], np.broadcast_to(mean, out[row].shape), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# P4 / P5: RMSNorm closed form and rotation invariants.

@pytest.mark.parametrize("scope", [0, 1])
def test_rmsnorm_closed_form_and_direction(scope):
    wl, g = tiny(heads=3)
    g.norm_scope = scope
    g.kv_frame_offset = 0
    inp = synth.make_inputs(wl)
    x = synth.bf16_bits_to_f64(inp.k[0, 0])          # token (t=0, y=0, x=0): no rotation
    out = oracle.norm_rope(g, inp.k, inp.gamma_k, False, [0])[0]
    D = g.head_dim
    groups = [slice(0, g.C)] if scope == 0 else [slice(h * D, (h + 1) * D) for h in range(g.heads)]
    for sl in groups:
        ms = np.mean(x[sl] ** 2)
        assert np.mean(out[sl] ** 2) == pytest.approx(1.0 / (1.0 + g.rms_eps / ms), rel=1e-12)
        assert np.all(out[sl] * x[sl] >= 0)
        cos = out[sl] @ x[sl] / np.linalg.norm(out[sl]) / np.linalg.norm(x[sl])
        assert cos == pytest.approx(1.0, abs=1e-13)


@pytest.mark.parametrize("scope", [0, 1])
def test_gain_scales_each_channel(scope):
    """Each channel's gain multiplies that channel after the norm, in both
    scopes (three heads, so the heads' gains differ)."""
    wl, g = tiny(heads=3)
    g.norm_scope = scope
    g.kv_frame_offset = 0                            # token (0, 0, 0): no rotation
    inp = synth.make_inputs(wl)
    gam = (1.0 + 0.25 * np.arange(g.C) / g.C).astype(np.float32)
    a = oracle.norm_rope(g, inp.k, inp.gamma_k, False, [0])[0]
    b = oracle.norm_rope(g, inp.k, gam, False, [0])[0]
    np.testing.assert_allclose(b, a * gam.astype(np.float64), rtol=1e-14, atol=0)


def _same_vector_everywhere(g, wl):
    inp = synth.make_inputs(wl)
    inp.k[:] = inp.k[:, :1]
    return inp


def test_rotation_preserves_pair_norms_and_splits_axes():
    wl, g = tiny(kv_frames=3, q_frames=3)
    inp = _same_vector_everywhere(g, wl)
    D = g.head_dim
    dh = 2 * (D // 6)
    dt = D - 2 * dh
    grp = {"t": slice(0, dt), "h": slice(dt, dt + dh), "w": slice(dt + dh, D)}

    def tok(t, y, x):
        return (t * g.grid_h + y) * g.grid_w + x

    base, dy, dx, dtt = oracle.norm_rope(g, inp.k, inp.gamma_k, False,
                                         [tok(0, 0, 0), tok(0, 5, 0), tok(0, 0, 7), tok(2, 0, 0)])
    for hd in range(g.heads):
        def part(vec, name):
            return vec[hd * D:(hd + 1) * D][grp[name]]
        for vec in (dy, dx, dtt):
            pn = np.hypot(vec[hd * D:(hd + 1) * D:2], vec[hd * D + 1:(hd + 1) * D:2])
            pb = np.hypot(base[hd * D:(hd + 1) * D:2], base[hd * D + 1:(hd + 1) * D:2])
            np.testing.assert_allclose(pn, pb, rtol=1e-13)
        # a move along one axis only turns that axis' pairs
        np.testing.assert_array_equal(part(dy, "t"), part(base, "t"))
        np.testing.assert_array_equal(part(dy, "w"), part(base, "w"))
        np.testing.assert_array_equal(part(dx, "t"), part(base, "t"))
        np.testing.assert_array_equal(part(dx, "h"), part(base, "h"))
        np.testing.assert_array_equal(part(dtt, "h"), part(base, "h"))
        np.testing.assert_array_equal(part(dtt, "w"), part(base, "w"))
        assert not np.allclose(part(dy, "h"), part(base, "h"))
        assert not np.allclose(part(dx, "w"), part(base, "w"))
        assert not np.allclose(part(dtt, "t"), part(base, "t"))


def _pair_angles(vec, ref):
    a = np.arctan2(vec[1::2], vec[0::2]) - np.arctan2(ref[1::2], ref[0::2])
    return np.angle(np.exp(1j * a))


def test_rotation_angle_is_linear_in_position_and_first_pair_turns_one_radian():
    wl, g = tiny(grid_w=32)
    inp = _same_vector_everywhere(g, wl)
    D = g.head_dim
    dh = 2 * (D // 6)
    dt = D - 2 * dh
    v0, v1, v2 = oracle.norm_rope(g, inp.k, inp.gamma_k, False, [0, 1, 2])   # x = 0, 1, 2
    a1 = _pair_angles(v1[:D], v0[:D])
    a2 = _pair_angles(v2[:D], v0[:D])
    np.testing.assert_allclose(np.angle(np.exp(1j * (a2 - 2 * a1))), 0.0, atol=1e-12)
    w0 = (dt + dh) // 2                         # first pair of the column axis
    assert a1[w0] == pytest.approx(1.0, abs=1e-12)
    # frequencies fall monotonically inside the column group
    grp = np.abs(a1[w0:])
    assert np.all(np.diff(grp) < 0)


def test_every_axis_follows_the_rope_frequency_schedule():
    """The RoPE reading: a step of one position along an axis of n dims turns
    that axis' pair j by 10000^(-2j/n) radians (the standard rotary frequencies
    per axis), with n = 44 for frames and 42 each for rows and columns at
    head_dim 128. Measured from the turn of each pair between neighbouring
    tokens that hold the same vector, and between tokens far apart on a
    grid wider than it is high (row and column come from the raster index)."""
    wl, g = tiny(kv_frames=2, q_frames=2, grid_w=32)
    inp = _same_vector_everywhere(g, wl)
    D = g.head_dim
    assert D == 128
    dims = {"t": 44, "h": 42, "w": 42}
    first = {"t": 0, "h": 22, "w": 43}           # first pair of each axis

    def tok(t, y, x):
        return (t * g.grid_h + y) * g.grid_w + x

    v0, vt, vh, vw, vfar = oracle.norm_rope(g, inp.k, inp.gamma_k, False,
                                            [tok(0, 3, 4), tok(1, 3, 4), tok(0, 4, 4), tok(0, 3, 5), tok(1, 11, 27)])
    for hd in range(g.heads):
        sl = slice(hd * D, (hd + 1) * D)
        for axis, vec in (("t", vt), ("h", vh), ("w", vw)):
            turn = _pair_angles(vec[sl], v0[sl])
            n = dims[axis]
            j = np.arange(n // 2)
            np.testing.assert_allclose(turn[first[axis] + j], 10000.0 ** (-2.0 * j / n), rtol=0, atol=1e-11)
        # (0, 3, 4) -> (1, 11, 27): 1 frame, 8 rows and 23 columns, angles modulo 2 pi
        turn = _pair_angles(vfar[sl], v0[sl])
        for axis, steps in (("t", 1), ("h", 8), ("w", 23)):
            n = dims[axis]
            j = np.arange(n // 2)
            np.testing.assert_allclose(np.exp(1j * turn[first[axis] + j]), np.exp(1j * steps * 10000.0 ** (-2.0 * j / n)),
                                       rtol=0, atol=1e-10)


def test_batch_entries_are_independent():
    """The entries of a batch do not interact: each entry of a batch-2 call
    gives the pooled values, selection and outputs of a batch-1 call on that
    entry alone (rows are numbered batch, then head, then query block)."""
    over = dict(heads=3, q_frames=1, kv_frames=2, local_range=3, topk=3)
    wl, g = tiny(batch=2, **over)
    inp = synth.make_inputs(wl)
    pq, pk, sel, out, _ = oracle.run(g, inp)
    _, g1 = tiny(batch=1, **over)
    per = g1.rows
    for b in range(2):
        one = synth.Inputs(q=inp.q[b:b + 1].copy(), k=inp.k[b:b + 1].copy(), v=inp.v[b:b + 1].copy(),
                           gamma_q=inp.gamma_q, gamma_k=inp.gamma_k)
        pq1, pk1, sel1, out1, _ = oracle.run(g1, one)
        np.testing.assert_array_equal(pq[b], pq1[0])
        np.testing.assert_array_equal(pk[b], pk1[0])
        r = slice(b * per, (b + 1) * per)
        np.testing.assert_array_equal(sel.row_len[r], sel1.row_len)
        np.testing.assert_array_equal(sel.cols[r], sel1.cols)
        np.testing.assert_array_equal(out[r], out1)
    assert not np.allclose(out[:per], out[per:])  # the two entries differ


def test_query_frames_are_the_last_frames_of_the_window():
    """Queries are the last q_frames of the KV window: a query token and the
    key token at the same place of the last KV frame, holding the same vector
    and gains, come out of the norm and rotation identical; the same vector at
    the same place of an earlier KV frame does not."""
    wl, g = tiny(q_frames=1, kv_frames=3, kv_frame_offset=4)
    inp = synth.make_inputs(wl)
    tpf = g.grid_h * g.grid_w
    inp.q[0, :tpf] = inp.k[0, 2 * tpf:3 * tpf]  # the query frame holds the last KV frame's vectors
    inp.k[0, :tpf] = inp.k[0, 2 * tpf:3 * tpf]  # and so does the first KV frame
    toks = np.arange(0, tpf, 37)
    qh = oracle.norm_rope(g, inp.q, inp.gamma_k, True, toks)
    k_last = oracle.norm_rope(g, inp.k, inp.gamma_k, False, 2 * tpf + toks)
    k_first = oracle.norm_rope(g, inp.k, inp.gamma_k, False, toks)
    np.testing.assert_array_equal(qh, k_last)
    assert not np.allclose(qh, k_first)


def test_scores_and_outputs_are_invariant_to_the_frame_offset():
    wl, g = tiny(q_frames=1, kv_frames=2, local_range=3)
    inp = synth.make_inputs(wl)
    res = []
    for off in (0, 7):
        g.kv_frame_offset = off
        pq, pk, sel, out, _ = oracle.run(g, inp)
        res.append((pq, pk, oracle.select(g, pq, pk, want_scores=True), out))
    (pq0, pk0, s0, o0), (pq1, pk1, s1, o1) = res
    fin = np.isfinite(s0.scores)
    np.testing.assert_allclose(s0.scores[fin], s1.scores[fin], rtol=0, atol=1e-9)
    np.testing.assert_array_equal(s0.cols, s1.cols)
    np.testing.assert_allclose(o0, o1, rtol=0, atol=1e-9)
    assert not np.allclose(pq0, pq1)            # the pooled vectors themselves do move


# --------------------------------------------------------------------------
# P6: pooled score closed form (block means of the per-token vectors).

def test_pooled_score_is_mean_of_token_dot_products():
    wl, g = tiny(grid_w=32, block_w=16, q_frames=1, kv_frames=2)
    inp = synth.make_inputs(wl)
    pq = oracle.pool(g, inp.q, inp.gamma_q, True)
    pk = oracle.pool(g, inp.k, inp.gamma_k, False)
    qt = oracle.norm_rope(g, inp.q, inp.gamma_q, True, np.arange(g.Lq))
    kt = oracle.norm_rope(g, inp.k, inp.gamma_k, False, np.arange(g.Lkv))
    D = g.head_dim
    for h in range(g.heads):
        for qb in range(g.nQB):
            tq = block_raster_tokens(g, qb)
            for kb in range(g.nKB):
                tk = block_raster_tokens(g, kb)
                dots = qt[tq, h * D:(h + 1) * D] @ kt[tk, h * D:(h + 1) * D].T
                assert pq[0, h, qb] @ pk[0, h, kb] == pytest.approx(dots.mean(), rel=1e-12, abs=1e-12)


# --------------------------------------------------------------------------
# Threshold reuse: on the scores it was recorded from, the recorded k-th best
# score keeps exactly the top-k selection (where the k-th and (k+1)-th scores
# differ); no threshold keeps the whole window; a threshold above every score
# keeps the single best block.

def test_threshold_of_a_selection_reproduces_it():
    wl, g = tiny(grid_h=48, grid_w=48, q_frames=1, kv_frames=2, local_range=5, topk=7, field=True,
                 unit_gain=False, seed=9)
    inp = synth.make_inputs(wl)
    pq = oracle.pool(g, inp.q, inp.gamma_q, True)
    pk = oracle.pool(g, inp.k, inp.gamma_k, False)
    sel = oracle.select(g, pq, pk, want_scores=True)
    th = oracle.kth_thresholds(g, sel.scores)
    again = oracle.threshold_select(g, sel.scores, th)
    sizes = oracle.window_sizes(g)
    checked = 0
    for r in range(g.rows):
        if sel.gap[r] <= 0:
            continue
        np.testing.assert_array_equal(again.row(r), sel.row(r))
        # the threshold is the k-th best score of the admissible set
        adm = np.sort(sel.scores[r][np.isfinite(sel.scores[r])])[::-1]
        assert adm.size == sizes[r % g.nQB]
        if g.topk < adm.size:
            assert th[r] == adm[g.topk - 1] and adm[g.topk] < th[r]
        else:
            assert th[r] == -np.inf
        checked += 1
    assert checked > g.rows // 2


def test_threshold_extremes_keep_all_or_the_best_block():
    wl, g = tiny(grid_h=32, grid_w=32, q_frames=1, kv_frames=2, local_range=3, topk=3, field=True,
                 unit_gain=False, seed=10)
    inp = synth.make_inputs(wl)
    pq = oracle.pool(g, inp.q, inp.gamma_q, True)
    pk = oracle.pool(g, inp.k, inp.gamma_k, False)
    sc = oracle.select(g, pq, pk, want_scores=True).scores
    sizes = oracle.window_sizes(g)
    every = oracle.threshold_select(g, sc, np.full(g.rows, -np.inf))
    none = oracle.threshold_select(g, sc, np.full(g.rows, np.inf))
    for r in range(g.rows):
        adm = np.flatnonzero(np.isfinite(sc[r]))
        assert every.row_len[r] == sizes[r % g.nQB]
        np.testing.assert_array_equal(every.row(r), adm)
        assert none.row_len[r] == 1
        assert none.row(r)[0] == adm[np.argmax(sc[r][adm])]
    # equal best scores: the lower block
    flat = np.where(np.isfinite(sc), 0.0, sc)
    tie = oracle.threshold_select(g, flat, np.full(g.rows, 1.0))
    for r in range(g.rows):
        assert tie.row(r).tolist() == [np.flatnonzero(np.isfinite(sc[r]))[0]]
