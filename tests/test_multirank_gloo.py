"""Multi-rank host logic on CPU: world_size-2 process groups over gloo.

* The head-sharded orchestration (block_sparse_video_lcsa_b200.sharded): each
  rank holds a slice of a layer's heads; the per-token sums of squares of the
  rank's slice are all-reduced, so every rank's norm sees the sums over all
  heads. The CUDA plan is replaced by a CPU stand-in of its two entry points
  (this tests the exchange, not the kernels, which tests/test_sharded_gpu.py
  checks against the oracle).
* bench.py's timing aggregation: the reported time is the slowest rank's.
"""
import os
import socket
import sys
import types

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, port):
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=WORLD,
                            timeout=__import__("datetime").timedelta(seconds=60))


class _CpuPlan:
    """CPU stand-in for a head-sharded plan: lcsa_sumsq and lcsa_forward_sharded
    on float tensors of the rank's head slice."""

    def __init__(self, batch, q_tokens, kv_tokens):
        self.cfg = types.SimpleNamespace(batch=batch)
        self.geometry = types.SimpleNamespace(q_tokens=q_tokens, kv_tokens=kv_tokens)
        self.seen = None
        self.calls = []

    def lcsa_sumsq(self, q, k, ssq, stream=None):
        self.calls.append("sumsq")
        ssq.copy_(torch.cat([(q.double() ** 2).sum(-1).reshape(-1), (k.double() ** 2).sum(-1).reshape(-1)]).float())
        return ssq

    def lcsa_forward_sharded(self, q, k, v, gamma_q, gamma_k, ssq, out, stream=None):
        self.calls.append("forward_sharded")
        self.seen = ssq.clone()
        return out


def _sharded_worker(rank, port, heads):
    _init(rank, port)
    try:
        from block_sparse_video_lcsa_b200.sharded import forward_heads_sharded, head_slices
        B, Lq, Lk, D = 2, 24, 40, 8
        rng = np.random.default_rng(11)  # the same full layer on every rank
        q = torch.from_numpy(rng.standard_normal((B, Lq, heads * D)).astype(np.float32))
        k = torch.from_numpy(rng.standard_normal((B, Lk, heads * D)).astype(np.float32))
        h0, h1 = head_slices(heads, WORLD)[rank]
        sl = slice(h0 * D, h1 * D)
        plan = _CpuPlan(B, Lq, Lk)
        qs, ks = q[..., sl].contiguous(), k[..., sl].contiguous()
        out = torch.empty_like(qs)
        ssq = torch.empty(B * (Lq + Lk), dtype=torch.float32)
        forward_heads_sharded(plan, qs, ks, ks, None, None, out, ssq=ssq)
        assert plan.calls == ["sumsq", "forward_sharded"], plan.calls
        want = torch.cat([(q.double() ** 2).sum(-1).reshape(-1), (k.double() ** 2).sum(-1).reshape(-1)])
        np.testing.assert_allclose(plan.seen.double().numpy(), want.numpy(), rtol=1e-6)
        # the rank's own sums alone are not the layer's (the exchange matters)
        own = torch.cat([(qs.double() ** 2).sum(-1).reshape(-1), (ks.double() ** 2).sum(-1).reshape(-1)])
        assert not np.allclose(own.numpy(), want.numpy(), rtol=1e-3)
    finally:
        dist.destroy_process_group()


def _timing_worker(rank, port):
    _init(rank, port)
    try:
        sys.path.insert(0, ROOT)
        import bench
        got = bench._max_over_ranks(1.5 + 2.0 * rank, "cpu")
        assert got == 1.5 + 2.0 * (WORLD - 1), got
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("heads", [2, 5])
def test_head_sharded_sums_are_all_reduced(heads):
    mp.spawn(_sharded_worker, args=(_free_port(), heads), nprocs=WORLD, join=True)


def test_bench_reports_the_slowest_rank():
    mp.spawn(_timing_worker, args=(_free_port(),), nprocs=WORLD, join=True)


def test_head_slices_cover_the_layer():
    from block_sparse_video_lcsa_b200.sharded import head_slices
    for heads in range(1, 17):
        for world in range(1, heads + 1):
            sl = head_slices(heads, world)
            assert sl[0][0] == 0 and sl[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(sl, sl[1:]))
            sizes = [h1 - h0 for h0, h1 in sl]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    for heads, world in ((3, 4), (12, 0), (1, 2)):
        with pytest.raises(ValueError):
            head_slices(heads, world)
