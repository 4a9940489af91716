"""Several lcsa_forward calls captured in one CUDA graph (the 30 attention
calls of a DiT chunk share one geometry) replay bit-identically to the same
calls made eagerly, and each replayed output matches the fp64 oracle of its
own inputs within the parity tolerance. lcsa_forward does no host
synchronisation and no allocation, so it can be captured; the plan is not
re-entrant, so the calls of one plan are ordered on one stream inside the
graph."""
import numpy as np
import pytest

import block_sparse_video_lcsa_b200 as L
import oracle
from block_sparse_video_lcsa_b200 import synth

from lcsa_harness import OUT_MAX_ABS, OUT_MEAN_ABS, block_rows_to_raster, torch_inputs

pytestmark = pytest.mark.gpu

_T = synth.WORKLOADS["tiny"]
WL = {
    "blocks128": _T.replace(heads=3, q_frames=1, kv_frames=3, grid_h=24, grid_w=48, block_w=16, local_range=3,
                            topk=5, kv_frame_offset=2, field=True, unit_gain=False),
    "blocks64": _T.replace(heads=2, q_frames=2, kv_frames=4, grid_h=32, grid_w=40, local_range=5, topk=9,
                           field=True, unit_gain=False),
    # 160 query-block pairs: the last pairs are cut and merged inside the graph
    "blocks64_cut_pairs": _T.replace(heads=8, q_frames=2, kv_frames=4, grid_h=32, grid_w=40, local_range=5, topk=9,
                                     field=True, unit_gain=False, seed=25),
}
LAYERS = 3


@pytest.mark.parametrize("name", list(WL))
def test_graph_replay_equals_eager_calls(name):
    import torch
    wl = WL[name]
    host = [synth.make_inputs(wl.replace(seed=10 + i)) for i in range(LAYERS)]
    layers = [torch_inputs(inp) for inp in host]
    plan = L.lcsa_plan_create(L.config_from_workload(wl), 0)
    try:
        eager = []
        for q, k, v, gq, gk in layers:
            out = torch.empty_like(q)
            plan.lcsa_forward(q, k, v, gq, gk, out)
            eager.append(out.clone())
        torch.cuda.synchronize()
        outs = [torch.full_like(t[0], float("nan")) for t in layers]
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                for (q, k, v, gq, gk), out in zip(layers, outs):
                    plan.lcsa_forward(q, k, v, gq, gk, out, side)
        for _ in range(2):   # replays are repeatable
            graph.replay()
        torch.cuda.synchronize()
        plan.lcsa_check_device_error()
        for a, b in zip(eager, outs):
            np.testing.assert_array_equal(a.view(torch.int16).cpu().numpy(), b.view(torch.int16).cpu().numpy())
        # each replayed layer against the oracle of its own inputs
        og = oracle.Geometry.from_workload(wl)
        D = og.head_dim
        for inp, out in zip(host, outs):
            _, _, _, ref, _ = oracle.run(og, inp)
            got = synth.bf16_bits_to_f64(out.view(torch.int16).cpu().numpy().view(np.uint16))
            err = np.concatenate([np.abs(got[b, tok, h * D:(h + 1) * D] - ref[n, i])
                                  for b, tok, h, n, i in block_rows_to_raster(og, np.arange(og.rows), ref)])
            assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (err.max(), err.mean())
        del graph
    finally:
        plan.destroy()
