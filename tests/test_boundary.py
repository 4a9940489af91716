"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, resolves the measured workloads to the geometry the oracle
derives independently, and maps every bad configuration to its status code
without aborting."""
import ctypes
import os
import re

import numpy as np
import pytest

import block_sparse_video_lcsa_b200 as L
import oracle
from block_sparse_video_lcsa_b200 import build as lcsa_build
from block_sparse_video_lcsa_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    lcsa_build.build()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(lcsa_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported_and_bound():
    names = declared_functions()
    assert len(names) >= 15
    raw = ctypes.CDLL(L.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    bound = {s[0] for s in L.SIGNATURES}
    assert bound == set(names)


def test_abi_version_and_status_strings():
    assert L.lcsa_abi_version() == L.ABI_VERSION == 2
    for code in range(9):
        assert L.lcsa_status_string(code).startswith("LCSA_")


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_resolved_geometry_matches_the_oracle(name):
    wl = synth.WORKLOADS[name]
    geo = L.lcsa_config_resolve(L.config_from_workload(wl))
    og = oracle.Geometry.from_workload(wl)
    sizes = oracle.window_sizes(og)
    assert geo.topk == og.topk
    assert geo.q_blocks == og.nQB and geo.kv_blocks == og.nKB
    assert geo.rows == og.rows
    assert geo.nnz == og.batch * og.heads * int(np.minimum(sizes, og.topk).sum())
    assert geo.min_window == sizes.min() and geo.max_window == sizes.max()
    assert geo.selected_flops == geo.nnz * 4 * og.nb * og.nb * og.head_dim


def test_head_dim_64_resolves():
    """head_dim 64 (the ABI's other head size): 24 / 20 / 20 RoPE dims, the
    softmax scale 1/8, the budget and window as for 128."""
    cfg = _cfg(head_dim=64)
    g = L.lcsa_config_resolve(cfg)
    ref = L.lcsa_config_resolve(_cfg())
    assert g.channels == cfg.heads * 64
    assert (g.topk, g.nnz, g.rows, g.max_window) == (ref.topk, ref.nnz, ref.rows, ref.max_window)
    assert g.selected_flops * 2 == ref.selected_flops


def test_stream_chunk_numbers():
    geo = L.lcsa_config_resolve(L.config_from_workload(synth.WORKLOADS["stream_768x1280"]))
    assert (geo.q_tokens, geo.kv_tokens, geo.q_blocks, geo.kv_blocks, geo.topk) == (7680, 23040, 60, 180, 60)
    assert geo.selected_flops == pytest.approx(362.4e9, rel=1e-3)


def _cfg(**over):
    c = L.config_from_workload(synth.WORKLOADS["tiny"])
    for k, v in over.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("over,code", [
    (dict(batch=0), L.LCSA_ERR_INVALID_ARG),
    (dict(heads=-1), L.LCSA_ERR_INVALID_ARG),
    (dict(local_range=4), L.LCSA_ERR_INVALID_ARG),
    (dict(local_range=-3), L.LCSA_ERR_INVALID_ARG),
    (dict(topk=-1), L.LCSA_ERR_INVALID_ARG),
    (dict(topk=0, sparse_ratio=0.0), L.LCSA_ERR_INVALID_ARG),
    (dict(topk=0, sparse_ratio=0.001), L.LCSA_ERR_INVALID_ARG),   # budget floors to 0 blocks
    (dict(norm_scope=2), L.LCSA_ERR_INVALID_ARG),
    (dict(rms_eps=0.0), L.LCSA_ERR_INVALID_ARG),
    (dict(softmax_scale=-1.0), L.LCSA_ERR_INVALID_ARG),
    (dict(kv_frame_offset=-1), L.LCSA_ERR_INVALID_ARG),
    (dict(q_frames=3), L.LCSA_ERR_SHAPE),                          # more query than KV frames
    (dict(grid_w=20), L.LCSA_ERR_SHAPE),                           # ragged block column
    (dict(grid_h=12), L.LCSA_ERR_SHAPE),                           # ragged block row
    (dict(block_t=2, q_frames=1, kv_frames=2), L.LCSA_ERR_SHAPE),
    (dict(head_dim=96), L.LCSA_ERR_UNSUPPORTED),                   # head_dim 64 and 128 only
    (dict(head_dim=256), L.LCSA_ERR_UNSUPPORTED),
    (dict(heads=17), L.LCSA_ERR_UNSUPPORTED),
    (dict(block_w=4), L.LCSA_ERR_UNSUPPORTED),                     # 32-token blocks
    (dict(block_h=16, block_w=8, grid_h=32), L.LCSA_ERR_UNSUPPORTED),  # 16 token rows per block
    (dict(heads=2, heads_total=1), L.LCSA_ERR_INVALID_ARG),        # a shard cannot hold more heads than its layer
])
def test_bad_configs_return_their_status(over, code):
    cfg = _cfg(**over)
    g = L.lcsa_geometry_t()
    st = L.lib().lcsa_config_resolve(ctypes.byref(cfg), ctypes.byref(g))
    assert st == code, L.lcsa_last_error_message()
    assert L.lcsa_last_error_message() != ""
    h = ctypes.c_void_p()
    assert L.lib().lcsa_plan_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == code
    assert h.value is None


@pytest.mark.parametrize("over,code", [
    (dict(topk=0, sparse_ratio=float("inf")), L.LCSA_ERR_INVALID_ARG),
    (dict(topk=0, sparse_ratio=float("nan")), L.LCSA_ERR_INVALID_ARG),
    (dict(rms_eps=float("inf")), L.LCSA_ERR_INVALID_ARG),
    (dict(rms_eps=float("nan")), L.LCSA_ERR_INVALID_ARG),
    (dict(grid_h=1 << 30, grid_w=1 << 30), L.LCSA_ERR_UNSUPPORTED),    # products beyond int64 if formed
    (dict(q_frames=1, kv_frames=1 << 30), L.LCSA_ERR_UNSUPPORTED),
    (dict(batch=1 << 30, heads=16), L.LCSA_ERR_UNSUPPORTED),
])
def test_extreme_values_are_refused_by_both_entry_paths(over, code):
    """Non-finite parameters and sizes whose products would overflow are
    refused before any product is formed, by the plan path and by the
    allocation-free path alike."""
    cfg = _cfg(**over)
    g = L.lcsa_geometry_t()
    assert L.lib().lcsa_config_resolve(ctypes.byref(cfg), ctypes.byref(g)) == code, L.lcsa_last_error_message()
    fake = 1 << 20
    assert L.lcsa_forward_noalloc(cfg, fake, fake, fake, fake, fake, fake, 0) == code, L.lcsa_last_error_message()


def test_huge_sparse_ratio_keeps_every_admissible_block():
    cfg = _cfg(topk=0, sparse_ratio=1e30, local_range=3)
    g = L.lcsa_config_resolve(cfg)
    assert g.topk == 1 << 30
    assert g.nnz == g.rows // g.q_blocks * sum(_window_sizes(cfg, g))


def _window_sizes(cfg, g):
    """Admissible blocks of every query block: frames x clipped row span x clipped column span."""
    r = (cfg.local_range - 1) // 2
    nh, nw = cfg.grid_h // cfg.block_h, cfg.grid_w // cfg.block_w
    out = []
    for qb in range(g.q_blocks):
        rem = qb % (nh * nw)
        hb, wb = divmod(rem, nw)
        rows = min(hb + r, nh - 1) - max(hb - r, 0) + 1
        cols = min(wb + r, nw - 1) - max(wb - r, 0) + 1
        out.append(cfg.kv_frames // cfg.block_t * rows * cols)
    return out


def test_window_too_large_for_the_selection_sort():
    cfg = _cfg(grid_h=8 * 40, grid_w=8 * 40, q_frames=1, kv_frames=3, local_range=0, topk=4)
    g = L.lcsa_geometry_t()
    assert L.lib().lcsa_config_resolve(ctypes.byref(cfg), ctypes.byref(g)) == L.LCSA_ERR_UNSUPPORTED


def test_null_arguments_never_crash():
    lib = L.lib()
    assert lib.lcsa_config_resolve(None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_plan_create(None, 0, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_forward(None, None, None, None, None, None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_forward_host(None, None, None, None, None, None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_check_device_error(None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_get_selection(None, None, 0, None, 0) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_get_intermediates(None, None, None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_plan_set_timing(None, 1) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_get_kernel_times(None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_forward_stream(None, None, None, None, None, None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_stream_push(None, None, None, None, 1, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_sumsq(None, None, None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_forward_sharded(None, None, None, None, None, None, None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_plan_set_threshold_reuse(None, 1) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_selection_nnz(None, None) == L.LCSA_ERR_INVALID_ARG
    lib.lcsa_plan_destroy(None)


def test_default_config_is_the_stream_chunk():
    c = L.lcsa_config_default()
    wl = synth.WORKLOADS["stream_768x1280"]
    for name in ("heads", "head_dim", "q_frames", "kv_frames", "grid_h", "grid_w", "block_t", "block_h", "block_w",
                 "local_range"):
        assert getattr(c, name) == getattr(wl, name), name
    assert c.sparse_ratio == 2.0 and c.topk == 0


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "liblcsa.so"))
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(L.LcsaLibraryMissing):
        L.lib()


def test_noalloc_entry_point_rejects_before_touching_a_device():
    big = L.config_from_workload(synth.WORKLOADS["stream_768x1280"])
    fake = 1 << 20   # never dereferenced: the size check comes first
    assert L.lcsa_forward_noalloc(big, fake, fake, fake, fake, fake, fake, 0) == L.LCSA_ERR_UNSUPPORTED
    assert L.lcsa_forward_noalloc(_cfg(local_range=2), fake, fake, fake, fake, fake, fake, 0) == \
        L.LCSA_ERR_INVALID_ARG
    assert L.lcsa_forward_noalloc(_cfg(grid_w=20), fake, fake, fake, fake, fake, fake, 0) == L.LCSA_ERR_SHAPE
    # head-sharded layers need a plan (lcsa_sumsq / lcsa_forward_sharded)
    assert L.lcsa_forward_noalloc(_cfg(heads=2, heads_total=4), fake, fake, fake, fake, fake, fake, 0) == \
        L.LCSA_ERR_UNSUPPORTED


@pytest.mark.parametrize("value", ["alloc", "alloc:0", "alloc:x", "launch:K9", "launch:", "oom", "copy:1"])
def test_a_malformed_fault_injection_value_is_refused(value, monkeypatch):
    """LCSA_FAULT is read before any device call, so a misspelt injection is
    refused (never silently ignored), with or without a GPU."""
    monkeypatch.setenv("LCSA_FAULT", value)
    cfg = _cfg()
    for create in (L.lib().lcsa_plan_create, L.lib().lcsa_plan_create_stream):
        h = ctypes.c_void_p()
        assert create(ctypes.byref(cfg), 0, ctypes.byref(h)) == L.LCSA_ERR_INVALID_ARG
        assert "LCSA_FAULT" in L.lcsa_last_error_message()
        assert h.value is None


@pytest.mark.parametrize("value", ["alloc:3", "launch:K1", "launch:K2", "launch:PAIR", "launch:K3", "launch:ROPE",
                                   "copy"])
def test_well_formed_fault_injection_values_pass_the_parser(value, monkeypatch):
    monkeypatch.setenv("LCSA_FAULT", value)
    cfg = _cfg()
    h = ctypes.c_void_p()
    st = L.lib().lcsa_plan_create(ctypes.byref(cfg), 0, ctypes.byref(h))
    # no GPU here: the plan fails at the device (or, on a GPU, at the injected allocation)
    assert st in (L.LCSA_ERR_CUDA, L.LCSA_ERR_OOM, L.LCSA_OK), st
    assert "not understood" not in L.lcsa_last_error_message()
    if st == L.LCSA_OK:
        L.lib().lcsa_plan_destroy(h)


def test_noalloc_status_call_without_any_call_is_clean():
    assert L.lcsa_noalloc_check_device_error(0) == L.LCSA_OK


def test_nvtx_ranges_compile(tmp_path):
    """The optional NVTX ranges (build --nvtx) compile in both entry-point
    files; the objects go to a temporary directory, the in-tree library is
    left as built."""
    import subprocess
    for f in ("lcsa_api.cu", "lcsa_noalloc.cu"):
        src = os.path.join(ROOT, "block_sparse_video_lcsa_b200", "csrc", f)
        cmd = [lcsa_build.NVCC] + lcsa_build.ARCH + lcsa_build.FLAGS + ["-DLCSA_NVTX", "-c", src, "-o",
                                                                       str(tmp_path / (f + ".o"))]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr[-2000:]


class _FakeTensor:
    """Just the attributes the binding's tensor checks read."""

    def __init__(self, dtype, shape, cuda_index=None, contiguous=True):
        import types
        self.dtype, self.shape, self._c = dtype, tuple(shape), contiguous
        self.is_cuda = cuda_index is not None
        self.device = types.SimpleNamespace(index=cuda_index, type="cuda" if self.is_cuda else "cpu")

    def is_contiguous(self):
        return self._c


def test_binding_refuses_tensors_it_cannot_pass_on():
    """dtype, shape, contiguity and device (the plan's GPU, or the host for the
    host-buffer call) are checked in Python before any C call: a tensor on
    another GPU would have the kernels read that GPU's memory."""
    import torch
    t = torch.bfloat16
    want = (1, 512, 256)
    L._expect_tensor(_FakeTensor(t, want, 1), t, want, "q", 1)
    L._expect_tensor(_FakeTensor(t, want), t, want, "q", "cpu")
    L._expect_tensor(12345, t, want, "q", 0)                       # raw addresses pass through
    for bad, dev in ((_FakeTensor(t, want, 0), 1),                 # another GPU
                     (_FakeTensor(t, want), 0),                    # host memory for a device argument
                     (_FakeTensor(t, want, 0), "cpu"),             # device memory for a host argument
                     (_FakeTensor(torch.float16, want, 0), 0),     # dtype
                     (_FakeTensor(t, (1, 512, 128), 0), 0),        # shape
                     (_FakeTensor(t, want, 0, contiguous=False), 0)):
        with pytest.raises(ValueError):
            L._expect_tensor(bad, t, want, "q", dev)
    # the host-buffer call checks before it reaches the library (here: a plan without a handle)
    plan = L.Plan.__new__(L.Plan)
    plan._h, plan.device = None, 0
    plan.cfg = L.config_from_workload(synth.WORKLOADS["tiny"])
    plan.geometry = L.lcsa_config_resolve(plan.cfg)
    g, c = plan.geometry, plan.cfg
    ok = [_FakeTensor(t, (c.batch, g.q_tokens, g.channels)), _FakeTensor(t, (c.batch, g.kv_tokens, g.channels)),
          _FakeTensor(t, (c.batch, g.kv_tokens, g.channels)), _FakeTensor(torch.float32, (g.channels,)),
          _FakeTensor(torch.float32, (g.channels,)), _FakeTensor(t, (c.batch, g.q_tokens, g.channels))]
    wrong = list(ok)
    wrong[1] = _FakeTensor(t, (c.batch, g.kv_tokens + 1, g.channels))
    with pytest.raises(ValueError):
        plan.lcsa_forward_host(*wrong, stream=0)
    wrong = list(ok)
    wrong[0] = _FakeTensor(t, (c.batch, g.q_tokens, g.channels), 0)
    with pytest.raises(ValueError):
        plan.lcsa_forward_host(*wrong, stream=0)
