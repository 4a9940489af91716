"""Seeded synthetic inputs for the LCSA call, and the named workloads.

This module holds no step of the attention method: it only draws numbers and
names problem sizes. Both the CUDA path (through the binding) and the CPU
oracle are fed from here, so the two always see identical bf16 bytes.

Recipe (all counter based, so any slice can be regenerated on its own):

* Uniform 64-bit words come from SplitMix64 (Steele, Lea, Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014): word i of stream s
  is mix64(s + (i + 1) * 0x9E3779B97F4A7C15).
* A uniform double is the top 53 bits of a word times 2**-53.
* Normals come in pairs from Box-Muller on words (2j, 2j+1):
  r = sqrt(-2 ln(1 - u0)), z0 = r cos(2 pi u1), z1 = r sin(2 pi u1).
* Values are formed in double, rounded to fp32 (round to nearest even) and
  then to bf16 (round to nearest even).
* The "smooth low-frequency field" that stands in for the spatial structure
  of real DiT activations is, per channel c of the heads*head_dim vector,
  F_c(t, y, x) = sum_{m<4} a_cm cos(2 pi (u_cm t / T + v_cm y / H' + w_cm x / W') + phi_cm)
  with u in {0, 1}, v, w in {0, 1, 2}, a ~ N(0, 0.5^2), phi ~ U[0, 2 pi).
  Q and K share one field (so pooled scores have spatial structure, like real
  attention maps), V gets its own.  The query frames are the last q_frames of
  the KV window, so a query at frame tq sits at t = kv_frames - q_frames + tq.

Streams: Q noise 4s+0, K noise 4s+1, V noise 4s+2, gains 4s+3 (first
heads*head_dim normals for the Q gain, next for the K gain), shared Q/K field
parameters 4s+4, V field parameters 4s+5.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Raw parameters of one LCSA call (no derived quantities)."""

    name: str
    batch: int
    heads: int
    head_dim: int
    q_frames: int
    kv_frames: int
    grid_h: int
    grid_w: int
    block_t: int
    block_h: int
    block_w: int
    local_range: int          # odd window diameter in blocks; 0 = unbounded
    topk: int                 # >0 explicit block budget; 0 = from sparse_ratio
    sparse_ratio: float
    kv_frame_offset: int
    field: bool               # add the smooth low-frequency field
    unit_gain: bool           # RMSNorm gains all 1 (else 1 + 0.05 N(0,1))
    seed: int = 0

    @property
    def q_tokens(self) -> int:
        return self.q_frames * self.grid_h * self.grid_w

    @property
    def kv_tokens(self) -> int:
        return self.kv_frames * self.grid_h * self.grid_w

    @property
    def channels(self) -> int:
        return self.heads * self.head_dim

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five problem sizes of the FlashVSR streaming DiT that the LCSA call is
# measured on. 768x1280 output -> 96x160 latent -> 48x80 tokens after the 2x2
# patchify; a stream chunk has 2 latent query frames and a 6-frame KV window
# (kv_ratio 3); the first chunk is 6-frame self-attention.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 128, 2, 2, 16, 16, 1, 8, 8, 3, 4, 0.0, 0,
                     field=False, unit_gain=True),
    "stream_768x1280": Workload("stream_768x1280", 1, 12, 128, 2, 6, 48, 80, 1, 8, 16, 11, 0, 2.0, 4,
                                field=True, unit_gain=False),
    "first_768x1280_sr2": Workload("first_768x1280_sr2", 1, 12, 128, 6, 6, 48, 80, 1, 8, 16, 11, 0, 2.0, 0,
                                   field=True, unit_gain=False),
    "first_768x1280_sr1.5": Workload("first_768x1280_sr1.5", 1, 12, 128, 6, 6, 48, 80, 1, 8, 16, 11, 0, 1.5, 0,
                                     field=True, unit_gain=False),
    "stream_768x1408": Workload("stream_768x1408", 1, 12, 128, 2, 6, 48, 88, 1, 8, 8, 9, 0, 2.0, 4,
                                field=True, unit_gain=False),
    "stream_2176x3840": Workload("stream_2176x3840", 1, 12, 128, 2, 6, 136, 240, 1, 8, 16, 11, 0, 2.0, 4,
                                 field=True, unit_gain=False),
}


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def uniform_words(stream: int, start: int, count: int) -> np.ndarray:
    """Words start .. start+count-1 of a SplitMix64 stream, as uint64."""
    idx = np.arange(start + 1, start + 1 + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        state = np.uint64(stream & 0xFFFFFFFFFFFFFFFF) + idx * _GOLDEN
        return _mix64(state)


def uniforms(stream: int, start: int, count: int) -> np.ndarray:
    w = uniform_words(stream, start, count)
    return (w >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normals(stream: int, start: int, count: int) -> np.ndarray:
    """Normals start .. start+count-1 of a stream (start must be even)."""
    assert start % 2 == 0
    npair = (count + 1) // 2
    u = uniforms(stream, start, 2 * npair).reshape(npair, 2)
    r = np.sqrt(-2.0 * np.log1p(-u[:, 0]))
    ang = 2.0 * np.pi * u[:, 1]
    z = np.empty((npair, 2), dtype=np.float64)
    z[:, 0] = r * np.cos(ang)
    z[:, 1] = r * np.sin(ang)
    return z.reshape(-1)[:count]


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """double -> fp32 (RNE) -> bf16 (RNE), returned as uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    rnd = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rnd) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _field_params(stream: int, channels: int):
    """Per (channel, term) integers u, v, w, amplitude a and phase phi."""
    uni = uniforms(stream, 0, channels * 4 * 4).reshape(channels, 4, 4)
    u = np.floor(uni[..., 0] * 2.0)
    v = np.floor(uni[..., 1] * 3.0)
    w = np.floor(uni[..., 2] * 3.0)
    phi = 2.0 * np.pi * uni[..., 3]
    amp = 0.5 * normals(stream, channels * 16 + (channels * 16) % 2, channels * 4).reshape(channels, 4)
    return u, v, w, amp, phi


def _field_rows(params, t_pos: int, frames: int, gh: int, gw: int) -> np.ndarray:
    """Field values of one latent frame, shape [gh*gw, channels]."""
    u, v, w, amp, phi = params
    ys = np.arange(gh, dtype=np.float64)
    xs = np.arange(gw, dtype=np.float64)
    # cos(A + B) with A over (y, c, m) and B over (x, c, m)
    a_arg = 2.0 * np.pi * (u[None] * t_pos / frames + v[None] * ys[:, None, None] / gh) + phi[None]
    b_arg = 2.0 * np.pi * w[None] * xs[:, None, None] / gw
    ca, sa = amp[None] * np.cos(a_arg), amp[None] * np.sin(a_arg)      # [gh, C, 4]
    cb, sb = np.cos(b_arg), np.sin(b_arg)                                # [gw, C, 4]
    out = np.einsum("ycm,xcm->yxc", ca, cb) - np.einsum("ycm,xcm->yxc", sa, sb)
    return out.reshape(gh * gw, -1)


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _tensor(wl: Workload, noise_stream: int, field_params, frames: int, t0: int) -> np.ndarray:
    """[batch, frames*gh*gw, channels] bf16 bits: noise plus optional field."""
    C = wl.channels
    per_frame = wl.grid_h * wl.grid_w
    out = np.empty((wl.batch, frames * per_frame, C), dtype=np.uint16)

    def one(job):
        b, f = job
        base = ((b * frames + f) * per_frame) * C
        x = normals(noise_stream, base, per_frame * C).reshape(per_frame, C)
        if field_params is not None:
            x = x + _field_rows(field_params, t0 + f, wl.kv_frames, wl.grid_h, wl.grid_w)
        out[b, f * per_frame:(f + 1) * per_frame] = to_bf16_bits(x)

    jobs = [(b, f) for b in range(wl.batch) for f in range(frames)]
    with _cf.ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(one, jobs))
    return out


@dataclasses.dataclass
class Inputs:
    """Host copies of one problem's inputs (bf16 as uint16 bits, gains fp32)."""

    q: np.ndarray        # [B, Lq, heads*d] uint16
    k: np.ndarray        # [B, Lkv, heads*d] uint16
    v: np.ndarray        # [B, Lkv, heads*d] uint16
    gamma_q: np.ndarray  # [heads*d] float32
    gamma_k: np.ndarray  # [heads*d] float32


def make_inputs(wl: Workload) -> Inputs:
    s = wl.seed
    C = wl.channels
    qk_field = _field_params(4 * s + 4, C) if wl.field else None
    v_field = _field_params(4 * s + 5, C) if wl.field else None
    q = _tensor(wl, 4 * s + 0, qk_field, wl.q_frames, wl.kv_frames - wl.q_frames)
    k = _tensor(wl, 4 * s + 1, qk_field, wl.kv_frames, 0)
    v = _tensor(wl, 4 * s + 2, v_field, wl.kv_frames, 0)
    if wl.unit_gain:
        gq = np.ones(C, dtype=np.float32)
        gk = np.ones(C, dtype=np.float32)
    else:
        g = normals(4 * s + 3, 0, 2 * C)
        gq = (1.0 + 0.05 * g[:C]).astype(np.float32)
        gk = (1.0 + 0.05 * g[C:]).astype(np.float32)
    return Inputs(q, k, v, gq, gk)
