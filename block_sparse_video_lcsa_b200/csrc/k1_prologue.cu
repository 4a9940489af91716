// K1: LCSA prologue. One pass over q and k that applies the QK RMSNorm, the
// gain, the factored 3D RoPE and the block mean-pooling, and writes q^ / k^
// in head-major, block-major order for the attention kernel.
//
// Pages: "Add FlashVSR contrib model ... on Neuron", Model Information (QK-norm,
// factored 3D RoPE) and Additional Information (the norm all-reduces across
// head-sharded ranks, so it spans all heads of a token); "FlashVSR: From 17.2
// FPS to 57.3 FPS at 768x1408", What Was Actually Slow (layout conversions,
// pooling and RoPE as separate glue kernels) and Rebuild sparse attention for
// Hopper (coalesced RoPE kernel, pooled keys).
//
// Work split: one CTA of 8 warps owns one block of 64 or 128 tokens; warp w
// handles tokens w, w+8, ... of the block, loading the next token while it
// works on the current one. A token's heads*128 bf16 values are read with
// 16-byte streaming loads, lane l taking 16-byte chunks l, l+32, ... so every
// load instruction of a warp covers 512 contiguous bytes. The sum of squares
// is a warp-shuffle reduction; the pooled sums are kept per warp in shared
// memory (each lane owns its slots) and reduced across the 8 warps in a fixed
// order, so the pooled values (and hence the block selection) are
// deterministic. Two CTAs fit on an SM, so a stream chunk's 240 blocks are all
// resident at once.
#include "lcsa_internal.h"

namespace lcsa {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

__global__ void rope_table_kernel(float2* tab, int Tkv, int gh, int gw, int t0, RopeSplit s) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int nt = Tkv * s.pairs_t, nh = gh * s.pairs_h, nw = gw * s.pairs_w;
  if (i >= nt + nh + nw) return;
  double pos, expo;
  if (i < nt) {
    pos = double(t0 + i / s.pairs_t);
    expo = 2.0 * (i % s.pairs_t) / s.dims_t;
  } else if (i < nt + nh) {
    const int k = i - nt;
    pos = double(k / s.pairs_h);
    expo = 2.0 * (k % s.pairs_h) / s.dims_h;
  } else {
    const int k = i - nt - nh;
    pos = double(k / s.pairs_w);
    expo = 2.0 * (k % s.pairs_w) / s.dims_w;
  }
  const double ang = pos * pow(10000.0, -expo);
  tab[i] = make_float2(float(cos(ang)), float(sin(ang)));
}

__device__ __forceinline__ uint4 load_stream(const uint4* p) { return __ldcs(p); }

__device__ __forceinline__ void unpack8(const uint4& r, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(h[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 r;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return r;
}

// CPL = 16-byte chunks per lane per token = ceil(heads * 16 / 32).
template <int CPL>
__device__ __forceinline__ void load_token(const uint4* src, int lane, int nchunks, uint4 (&raw)[CPL]) {
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const int c = i * 32 + lane;
    raw[i] = make_uint4(0u, 0u, 0u, 0u);
    if (c < nchunks) raw[i] = load_stream(src + c);
  }
}

template <int CPL>
__global__ void __launch_bounds__(kThreads, 2) prologue_kernel(const K1Params p) {
  extern __shared__ float red[];  // [kWarps][C]
  const Grid& g = p.g;
  const int n_qtot = g.B * g.nQB;
  const bool is_q = int(blockIdx.x) < n_qtot;
  const int bg = is_q ? int(blockIdx.x) : int(blockIdx.x) - n_qtot;
  const int nblk = is_q ? g.nQB : g.nKB;
  const int b = bg / nblk, blk = bg % nblk;
  const __nv_bfloat16* x = is_q ? p.q : p.k;
  const float* gamma = is_q ? p.gamma_q : p.gamma_k;
  __nv_bfloat16* xhat = is_q ? p.qhat : p.khat;
  float* pooled = is_q ? p.pooled_q : p.pooled_k;
  const int64_t L = is_q ? g.Lq : g.Lkv;
  const int tshift = is_q ? (g.Tkv - g.Tq) : 0;

  const int tb = blk / g.bpf, rem = blk % g.bpf;
  const int t0 = tb * g.bt, y0 = (rem / g.nWb) * g.bh, x0 = (rem % g.nWb) * g.bw;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunks = g.C / 8;
  const int plane = g.bh * g.bw;
  constexpr int PT = 22, PH = 21;  // RoPE pairs on the frame / row axes (head_dim 128)

  // this lane's pooled partial sums live in its own slots of red[warp][.]
  float* mine = red + warp * g.C;
#pragma unroll
  for (int c4 = 0; c4 < CPL; ++c4) {
    const int c = c4 * 32 + lane;
    if (c < nchunks) {
      reinterpret_cast<float4*>(mine + c * 8)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      reinterpret_cast<float4*>(mine + c * 8)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }

  auto token_src = [&](int i, int& t, int& y, int& xc) {
    t = t0 + i / plane;
    y = y0 + (i / g.bw) % g.bh;
    xc = x0 + i % g.bw;
    const int64_t tok = (int64_t(t) * g.gh + y) * g.gw + xc;
    return reinterpret_cast<const uint4*>(x + (int64_t(b) * L + tok) * g.C);
  };

  const int jb = 4 * (lane & 15);  // first RoPE pair of this lane (same in every head)
  uint4 nxt[CPL];
  int nt = 0, ny = 0, nx = 0;
  if (warp < g.nb) load_token<CPL>(token_src(warp, nt, ny, nx), lane, nchunks, nxt);
  for (int i = warp; i < g.nb; i += kWarps) {
    uint4 raw[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) raw[c] = nxt[c];
    const int t = nt, y = ny, xc = nx;
    if (i + kWarps < g.nb) load_token<CPL>(token_src(i + kWarps, nt, ny, nx), lane, nchunks, nxt);
    // RMSNorm scale(s)
    float rs[CPL];
    if (p.norm_scope == 0) {
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        float f[8];
        unpack8(raw[c], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float r = rsqrtf(ss * (1.0f / float(g.C)) + p.eps);
#pragma unroll
      for (int c = 0; c < CPL; ++c) rs[c] = r;
    } else {
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        float f[8];
        unpack8(raw[c], f);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        rs[c] = rsqrtf(ss * (1.0f / float(kHeadDim)) + p.eps);
      }
    }
    // cos/sin of this lane's four pairs at this token's position
    float2 cs[4];
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      const int j = jb + qd;
      if (j < PT)
        cs[qd] = p.rope[(tshift + t) * PT + j];
      else if (j < PT + PH)
        cs[qd] = p.rope[p.rope_h_off + y * PH + (j - PT)];
      else
        cs[qd] = p.rope[p.rope_w_off + xc * (kHeadDim / 2 - PT - PH) + (j - PT - PH)];
    }
#pragma unroll
    for (int c4 = 0; c4 < CPL; ++c4) {
      const int c = c4 * 32 + lane;
      if (c >= nchunks) continue;
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(gamma + c * 8));
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(gamma + c * 8 + 4));
      const float gm[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      float f[8], o[8];
      unpack8(raw[c4], f);
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) {
        const float a = f[2 * qd] * rs[c4] * gm[2 * qd];
        const float bq = f[2 * qd + 1] * rs[c4] * gm[2 * qd + 1];
        o[2 * qd] = a * cs[qd].x - bq * cs[qd].y;
        o[2 * qd + 1] = a * cs[qd].y + bq * cs[qd].x;
      }
      float4* acc = reinterpret_cast<float4*>(mine + c * 8);
      float4 a0 = acc[0], a1 = acc[1];
      a0.x += o[0]; a0.y += o[1]; a0.z += o[2]; a0.w += o[3];
      a1.x += o[4]; a1.y += o[5]; a1.z += o[6]; a1.w += o[7];
      acc[0] = a0;
      acc[1] = a1;
      const int head = c >> 4, dd = (c & 15) * 8;
      uint4* dst = reinterpret_cast<uint4*>(
          xhat + (((int64_t(b) * g.Hn + head) * nblk + blk) * g.nb + i) * kHeadDim + dd);
      *dst = pack8(o);
    }
  }

  // warp partials -> block mean, summed over warps in a fixed order
  __syncthreads();
  const float inv_nb = 1.0f / float(g.nb);
  for (int e = threadIdx.x; e < g.C; e += kThreads) {
    float s = red[e];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) s += red[w * g.C + e];
    const int head = e / kHeadDim, dd = e % kHeadDim;
    pooled[((int64_t(b) * g.Hn + head) * nblk + blk) * kHeadDim + dd] = s * inv_nb;
  }
}

template <int CPL>
cudaError_t launch_cpl(const K1Params& p, cudaStream_t s) {
  const int nblocks = p.g.B * (p.g.nQB + p.g.nKB);
  const size_t smem = size_t(kWarps) * p.g.C * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(prologue_kernel<CPL>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  prologue_kernel<CPL><<<nblocks, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rope_table(float2* table, int Tkv, int gh, int gw, int t0, int d, cudaStream_t s) {
  const RopeSplit rs = rope_split(d);
  const int n = Tkv * rs.pairs_t + gh * rs.pairs_h + gw * rs.pairs_w;
  rope_table_kernel<<<(n + 255) / 256, 256, 0, s>>>(table, Tkv, gh, gw, t0, rs);
  return cudaGetLastError();
}

cudaError_t launch_prologue(const K1Params& p, cudaStream_t s) {
  switch ((p.g.Hn + 1) / 2) {
    case 1: return launch_cpl<1>(p, s);
    case 2: return launch_cpl<2>(p, s);
    case 3: return launch_cpl<3>(p, s);
    case 4: return launch_cpl<4>(p, s);
    case 5: return launch_cpl<5>(p, s);
    case 6: return launch_cpl<6>(p, s);
    case 7: return launch_cpl<7>(p, s);
    case 8: return launch_cpl<8>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace lcsa
