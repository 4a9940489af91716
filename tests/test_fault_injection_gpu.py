"""Error paths forced from the host (LCSA_FAULT, read when a plan is created;
no GPU fault is involved). The pages' standard is to fail loudly rather than
fall back ("FlashVSR: From 17.2 FPS to 57.3 FPS at 768x1408", Reproducibility
And Profiling: a run that silently falls back is a failed run):

* a device allocation failing at each position of a plan's creation returns
  LCSA_ERR_OOM and frees what was already allocated;
* a failed kernel launch (each kernel of the call) or host copy returns
  LCSA_ERR_CUDA naming it;
* afterwards the CUDA context is still usable: a clean plan passes parity.
"""
import numpy as np
import pytest

import block_sparse_video_lcsa_b200 as L
import oracle
from block_sparse_video_lcsa_b200 import synth

from lcsa_harness import OUT_MAX_ABS, OUT_MEAN_ABS, check_output, run_gpu, torch_inputs

pytestmark = pytest.mark.gpu

_T = synth.WORKLOADS["tiny"]
BLOCKS64 = _T.replace(heads=2, q_frames=2, kv_frames=4, grid_h=32, grid_w=40, local_range=5, topk=9, field=True,
                      unit_gain=False, seed=3)
BLOCKS128 = _T.replace(heads=3, q_frames=1, kv_frames=3, grid_h=24, grid_w=48, block_w=16, local_range=3, topk=5,
                       kv_frame_offset=2, field=True, unit_gain=False)


def _parity(wl):
    """A clean plan on the same context still matches the oracle (all rows)."""
    inp = synth.make_inputs(wl)
    og = oracle.Geometry.from_workload(wl)
    gpu = run_gpu(wl, inp)
    _, _, sel, ref, _ = oracle.run(og, inp)
    np.testing.assert_array_equal(gpu.row_ptr.astype(np.int64), sel.csr()[0])
    mx, mean = check_output(og, gpu, np.arange(og.rows), ref)
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, (mx, mean)


@pytest.mark.parametrize("kind", ["plan", "host_io", "stream"])
def test_every_allocation_failure_is_reported_and_freed(kind, monkeypatch):
    import torch
    wl = synth.WORKLOADS["stream_768x1280"]    # allocations of tens of MB: a leak would show
    cfg = L.config_from_workload(wl, host_io=1 if kind == "host_io" else 0)
    create = L.lcsa_plan_create_stream if kind == "stream" else L.lcsa_plan_create
    monkeypatch.delenv("LCSA_FAULT", raising=False)
    create(cfg, 0).destroy()                   # kernels' modules loaded before the baseline
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(0)[0]
    n = 1
    while True:
        monkeypatch.setenv("LCSA_FAULT", "alloc:%d" % n)
        try:
            plan = create(cfg, 0)
        except L.LcsaError as e:
            assert e.status == L.LCSA_ERR_OOM and "injected" in str(e), str(e)
            n += 1
            continue
        plan.destroy()                         # n is past the last allocation
        break
    monkeypatch.delenv("LCSA_FAULT")
    assert n > 10, "only %d allocation positions" % (n - 1)
    free1 = torch.cuda.mem_get_info(0)[0]
    assert abs(free1 - free0) <= 8 << 20, "device memory not returned: %d bytes" % (free0 - free1)


@pytest.mark.parametrize("kernel,wl", [("K1", BLOCKS128), ("K2", BLOCKS128), ("K3", BLOCKS128),
                                       ("PAIR", BLOCKS64), ("K3", BLOCKS64)])
def test_a_failed_launch_is_reported_and_the_context_stays_usable(kernel, wl, monkeypatch):
    import torch
    monkeypatch.setenv("LCSA_FAULT", "launch:" + kernel)
    plan = L.lcsa_plan_create(L.config_from_workload(wl), 0)
    monkeypatch.delenv("LCSA_FAULT")
    try:
        q, k, v, gq, gk = torch_inputs(synth.make_inputs(wl))
        out = torch.empty_like(q)
        with pytest.raises(L.LcsaError) as ei:
            plan.lcsa_forward(q, k, v, gq, gk, out)
        assert ei.value.status == L.LCSA_ERR_CUDA and "injected" in str(ei.value), str(ei.value)
        plan.lcsa_check_device_error()         # whatever did launch ran cleanly
    finally:
        plan.destroy()
    _parity(wl)


def test_a_failed_rope_table_launch_of_a_stream_push_is_reported(monkeypatch):
    import torch
    wl = BLOCKS128
    monkeypatch.setenv("LCSA_FAULT", "launch:ROPE")
    plan = L.lcsa_plan_create_stream(L.config_from_workload(wl), 0)
    monkeypatch.delenv("LCSA_FAULT")
    try:
        _, k, v, _, gk = torch_inputs(synth.make_inputs(wl))
        with pytest.raises(L.LcsaError) as ei:
            plan.lcsa_stream_push(k, v, gk, wl.kv_frames)
        assert ei.value.status == L.LCSA_ERR_CUDA and "rope" in str(ei.value)
    finally:
        plan.destroy()
    _parity(wl)


def test_a_failed_host_copy_is_reported(monkeypatch):
    import torch
    wl = BLOCKS128
    monkeypatch.setenv("LCSA_FAULT", "copy")
    plan = L.lcsa_plan_create(L.config_from_workload(wl, host_io=1), 0)
    monkeypatch.delenv("LCSA_FAULT")
    try:
        inp = synth.make_inputs(wl)
        host = [t.cpu().pin_memory() for t in torch_inputs(inp)]
        out = torch.empty_like(host[0]).pin_memory()
        with pytest.raises(L.LcsaError) as ei:
            plan.lcsa_forward_host(*host, out)
        assert ei.value.status == L.LCSA_ERR_CUDA and "host-to-device" in str(ei.value)
    finally:
        plan.destroy()
    _parity(wl)
