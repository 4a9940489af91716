"""Head-sharded LCSA layers over torch.distributed.

The tensor-parallel form of the pages ("Add FlashVSR contrib model with video
super-resolution on Neuron", Model Information and Additional Information):
each rank holds a slice of a layer's heads, and the QK RMSNorm, whose mean runs
over all heads of a token, needs one exchange: an all-reduce (sum) of the
per-token sums of squares, 4 bytes per token and tensor. Everything else (the
rotation, pooling, block selection and attention of the rank's heads) is
independent per rank.

Per call, on the current torch stream of each rank:
  1. ``plan.lcsa_sumsq``: the sums of squares of the rank's own q and k channels;
  2. ``torch.distributed.all_reduce`` of those sums (NCCL between GPUs);
  3. ``plan.lcsa_forward_sharded``: the LCSA call with the reduced sums.

The plans are made with ``heads`` = the rank's heads and ``heads_total`` = the
layer's heads (``head_slices`` gives the usual contiguous split). Head-scope
norm needs no exchange and uses ``lcsa_forward`` directly.
"""
from __future__ import annotations


def head_slices(heads_total: int, world: int):
    """Contiguous head ranges [h0, h1) of `world` ranks, sizes differing by at
    most one; every rank holds at least one head."""
    if world < 1 or heads_total < world:
        raise ValueError("cannot split %d heads over %d ranks (each rank needs at least one head)"
                         % (heads_total, world))
    base, extra = divmod(heads_total, world)
    out, h0 = [], 0
    for r in range(world):
        h1 = h0 + base + (1 if r < extra else 0)
        out.append((h0, h1))
        h0 = h1
    return out


def sumsq_buffer(plan, device):
    """A device buffer for the per-token sums of `plan` (q tokens, then k tokens)."""
    import torch
    g, c = plan.geometry, plan.cfg
    return torch.empty(c.batch * (g.q_tokens + g.kv_tokens), dtype=torch.float32, device=device)


def forward_heads_sharded(plan, q, k, v, gamma_q, gamma_k, out, ssq=None, group=None):
    """One head-sharded LCSA call on this rank: q, k, v, out, gains are the
    rank's head slice; every rank of `group` calls this with the same chunk.
    Without an initialised process group (or with one rank) the sums are the
    rank's own, which is the whole layer when heads == heads_total."""
    import torch.distributed as dist

    if ssq is None:
        ssq = sumsq_buffer(plan, q.device)
    plan.lcsa_sumsq(q, k, ssq)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(ssq, op=dist.ReduceOp.SUM, group=group)
    plan.lcsa_forward_sharded(q, k, v, gamma_q, gamma_k, ssq, out)
    return out
