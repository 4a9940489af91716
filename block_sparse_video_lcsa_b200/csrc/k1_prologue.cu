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
// Work split: a persistent grid of one CTA (8 warps) per SM walks the q and
// k blocks blockIdx.x, blockIdx.x + gridDim.x, ... A block is bt * bh rows of
// bw tokens, and each row is one contiguous run of bw * heads * 128 bf16 in
// the raster input, so one thread streams rows into a ring of shared-memory
// stages with bulk asynchronous copies (cp.async.bulk, completion counted on
// an mbarrier), several rows ahead and across block boundaries, while the
// warps work on the oldest stage: warp w takes tokens w, w+8, ... of the row,
// lane l the 16-byte chunks l, l+32, ... of a token (conflict-free shared
// loads), so each lane always holds the same channels. The gain and the
// pooled sums therefore live in registers for the whole block; the sum of
// squares is a warp-shuffle reduction; at the end of a block the 8 warps'
// partial sums are added in a fixed order, so the pooled values (and hence
// the block selection) are deterministic. q^ / k^ are written with 16-byte
// stores, every store instruction of a warp covering whole 256-byte rows of
// two heads.
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

// bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 word.
// Done with integer shifts and masks, which leaves the conversion unit free.
__device__ __forceinline__ void unpack8(const uint4& r, float (&f)[8]) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
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
constexpr int kMaxStages = 4;
constexpr uint32_t kSmemBudget = 220 * 1024;
constexpr uint32_t kBarBytes = 128;  // mbarriers of the ring
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; false once the wall-clock limit has passed.
__device__ __noinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}
// One row of the raster input (contiguous, 16-byte aligned, a multiple of 16
// bytes) into shared memory; completion is counted in bytes on `bar`.
__device__ __forceinline__ void bulk_row(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Block number bid of the combined list (B * nQB query blocks, then B * nKB
// key blocks) -> which tensor, batch element, block and its first token.
struct BlockRef {
  bool is_q;
  int b, blk, nblk, t0, y0, x0;
};
__device__ __forceinline__ BlockRef block_ref(const Grid& g, int bid) {
  BlockRef r;
  const int n_qtot = g.B * g.nQB;
  r.is_q = bid < n_qtot;
  const int bg = r.is_q ? bid : bid - n_qtot;
  r.nblk = r.is_q ? g.nQB : g.nKB;
  r.b = bg / r.nblk;
  r.blk = bg % r.nblk;
  const int tb = r.blk / g.bpf, rem = r.blk % g.bpf;
  r.t0 = tb * g.bt;
  r.y0 = (rem / g.nWb) * g.bh;
  r.x0 = (rem % g.nWb) * g.bw;
  return r;
}

// CPL = 16-byte chunks per lane per token = ceil(heads * 16 / 32); FULL: every
// lane's CPL chunks exist (even head count); HEAD: per-head norm scope.
template <int CPL, bool FULL, bool HEAD>
__global__ void __launch_bounds__(kThreads, 1) prologue_kernel(const K1Params p, int stages, uint32_t row_bytes) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Grid& g = p.g;
  const uint32_t bars = smem_u32(smem);
  uint8_t* ring = smem + kBarBytes;
  float* red = reinterpret_cast<float*>(ring + size_t(stages) * row_bytes);  // [kWarps][C]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunks = g.C / 8;
  const int R = g.bt * g.bh;  // rows per block
  const int total = g.B * (g.nQB + g.nKB);
  const int my_blocks = (total - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x);
  const int my_rows = my_blocks * R;
  constexpr int PT = 22, PH = 21;  // RoPE pairs on the frame / row axes (head_dim 128)

  // source of the CTA's row number gi (its blocks' rows, in order)
  auto row_src = [&](int gi) -> const void* {
    const BlockRef br = block_ref(g, int(blockIdx.x) + (gi / R) * int(gridDim.x));
    const int r = gi % R;
    const int64_t tok = (int64_t(br.t0 + r / g.bh) * g.gh + br.y0 + r % g.bh) * g.gw + br.x0;
    const __nv_bfloat16* x = br.is_q ? p.q : p.k;
    const int64_t L = br.is_q ? g.Lq : g.Lkv;
    return x + (int64_t(br.b) * L + tok) * g.C;
  };
  auto issue = [&](int gi) {
    const int s = gi % stages;
    bulk_row(smem_u32(ring + size_t(s) * row_bytes), row_src(gi), row_bytes, bars + 8 * s);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bars + 8 * s));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int gi = 0; gi < stages && gi < my_rows; ++gi) issue(gi);

  const int jb = 4 * (lane & 15);  // first RoPE pair of this lane (same in every head)
  float gm[CPL][8], acc[CPL][8];
  int gi = 0;
  bool ok = true;
  for (int kb = 0; kb < my_blocks && ok; ++kb) {
    const BlockRef br = block_ref(g, int(blockIdx.x) + kb * int(gridDim.x));
    const float* gamma = br.is_q ? p.gamma_q : p.gamma_k;
    __nv_bfloat16* xhat = br.is_q ? p.qhat : p.khat;
    float* pooled = br.is_q ? p.pooled_q : p.pooled_k;
    const int tshift = br.is_q ? (g.Tkv - g.Tq) : 0;
#pragma unroll
    for (int c4 = 0; c4 < CPL; ++c4) {
      const int c = c4 * 32 + lane;
      float4 g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0;
      if (c < nchunks) {
        g0 = __ldg(reinterpret_cast<const float4*>(gamma + c * 8));
        g1 = __ldg(reinterpret_cast<const float4*>(gamma + c * 8 + 4));
      }
      gm[c4][0] = g0.x; gm[c4][1] = g0.y; gm[c4][2] = g0.z; gm[c4][3] = g0.w;
      gm[c4][4] = g1.x; gm[c4][5] = g1.y; gm[c4][6] = g1.z; gm[c4][7] = g1.w;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[c4][e] = 0.f;
    }
    for (int r = 0; r < R; ++r, ++gi) {
      const int s = gi % stages;
      const bool arrived = mbar_wait_bounded(bars + 8 * s, uint32_t(gi / stages) & 1u);
      const int t = br.t0 + r / g.bh, y = br.y0 + r % g.bh;
      const uint4* row = reinterpret_cast<const uint4*>(ring + size_t(s) * row_bytes);
      for (int i = warp; i < g.bw; i += kWarps) {
        const int xc = br.x0 + i;
        uint4 raw[CPL];
#pragma unroll
        for (int c4 = 0; c4 < CPL; ++c4) {
          const int c = c4 * 32 + lane;
          raw[c4] = (FULL || c < nchunks) ? row[i * nchunks + c] : make_uint4(0u, 0u, 0u, 0u);
        }
        // cos/sin of this lane's four pairs at this token's position
        float2 cs[4];
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          const int j = jb + qd;
          const int idx = j < PT        ? (tshift + t) * PT + j
                          : j < PT + PH ? p.rope_h_off + y * PH + (j - PT)
                                        : p.rope_w_off + xc * (kHeadDim / 2 - PT - PH) + (j - PT - PH);
          cs[qd] = __ldg(p.rope + idx);
        }
        // RMSNorm scale(s), folded into the rotation: x^ = rot(rs * (x * gamma))
        float ca[HEAD ? CPL : 1][4], cb[HEAD ? CPL : 1][4];
        if (!HEAD) {
          float ss = 0.f;
#pragma unroll
          for (int c4 = 0; c4 < CPL; ++c4) {
            float f[8];
            unpack8(raw[c4], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          const float rr = rsqrtf(ss * (1.0f / float(g.C)) + p.eps);
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            ca[0][qd] = rr * cs[qd].x;
            cb[0][qd] = rr * cs[qd].y;
          }
        } else {
#pragma unroll
          for (int c4 = 0; c4 < (HEAD ? CPL : 1); ++c4) {
            float f[8];
            unpack8(raw[c4], f);
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float rr = rsqrtf(ss * (1.0f / float(kHeadDim)) + p.eps);
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
              ca[c4][qd] = rr * cs[qd].x;
              cb[c4][qd] = rr * cs[qd].y;
            }
          }
        }
        const int ti = r * g.bw + i;  // token index inside the block
#pragma unroll
        for (int c4 = 0; c4 < CPL; ++c4) {
          const int c = c4 * 32 + lane;
          if (!FULL && c >= nchunks) continue;
          const int cc = HEAD ? c4 : 0;
          float f[8], o[8];
          unpack8(raw[c4], f);
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            const float u0 = f[2 * qd] * gm[c4][2 * qd];
            const float u1 = f[2 * qd + 1] * gm[c4][2 * qd + 1];
            o[2 * qd] = fmaf(u0, ca[cc][qd], -u1 * cb[cc][qd]);
            o[2 * qd + 1] = fmaf(u0, cb[cc][qd], u1 * ca[cc][qd]);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[c4][e] += o[e];
          const int head = c >> 4, dd = (c & 15) * 8;
          uint4* dst = reinterpret_cast<uint4*>(
              xhat + (((int64_t(br.b) * g.Hn + head) * br.nblk + br.blk) * g.nb + ti) * kHeadDim + dd);
          *dst = pack8(o);
        }
      }
      // every warp is done with stage s (and agrees on whether the row arrived)
      if (__syncthreads_or(!arrived)) {
        ok = false;
        break;
      }
      if (threadIdx.x == 0 && gi + stages < my_rows) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(gi + stages);
      }
    }
    if (!ok) break;
    // warp partials -> block mean, summed over warps in a fixed order
    float* mine = red + warp * g.C;
#pragma unroll
    for (int c4 = 0; c4 < CPL; ++c4) {
      const int c = c4 * 32 + lane;
      if (c < nchunks) {
        reinterpret_cast<float4*>(mine + c * 8)[0] = make_float4(acc[c4][0], acc[c4][1], acc[c4][2], acc[c4][3]);
        reinterpret_cast<float4*>(mine + c * 8)[1] = make_float4(acc[c4][4], acc[c4][5], acc[c4][6], acc[c4][7]);
      }
    }
    __syncthreads();
    const float inv_nb = 1.0f / float(g.nb);
    for (int e = threadIdx.x; e < g.C; e += kThreads) {
      float sum = red[e];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) sum += red[w * g.C + e];
      const int head = e / kHeadDim, dd = e % kHeadDim;
      pooled[((int64_t(br.b) * g.Hn + head) * br.nblk + br.blk) * kHeadDim + dd] = sum * inv_nb;
    }
    __syncthreads();  // red is rewritten by the next block
  }
  if (!ok && threadIdx.x == 0) {
    // a row never arrived: record it, then give the copies still in flight a
    // bounded chance to land before the CTA (and its shared memory) goes away
    if (atomicCAS(p.err, kDevErrNone, kDevErrTimeout) == kDevErrNone) {
      p.err[1] = 1;
      p.err[2] = blockIdx.x;
    }
    for (int k = gi; k < gi + stages && k < my_rows; ++k)
      (void)mbar_wait_bounded(bars + 8 * (k % stages), uint32_t(k / stages) & 1u);
  }
}

template <int CPL, bool FULL, bool HEAD>
cudaError_t launch_cpl(const K1Params& p, cudaStream_t s) {
  const int nblocks = p.g.B * (p.g.nQB + p.g.nKB);
  if (nblocks <= 0) return cudaSuccess;
  const uint32_t row_bytes = uint32_t(p.g.bw) * uint32_t(p.g.C) * 2u;
  const uint32_t red_bytes = uint32_t(kWarps) * uint32_t(p.g.C) * 4u;
  int stages = int((kSmemBudget - kBarBytes - red_bytes) / row_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2 || p.num_sms <= 0) return cudaErrorInvalidValue;
  const size_t smem = kBarBytes + size_t(stages) * row_bytes + red_bytes;
  cudaError_t e = cudaFuncSetAttribute(prologue_kernel<CPL, FULL, HEAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int grid = nblocks < p.num_sms ? nblocks : p.num_sms;
  prologue_kernel<CPL, FULL, HEAD><<<grid, kThreads, smem, s>>>(p, stages, row_bytes);
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
  const bool full = p.g.Hn % 2 == 0, head = p.norm_scope != 0;
#define LCSA_K1_CASE(n)                                                              \
  case n:                                                                            \
    if (full) return head ? launch_cpl<n, true, true>(p, s) : launch_cpl<n, true, false>(p, s); \
    return head ? launch_cpl<n, false, true>(p, s) : launch_cpl<n, false, false>(p, s);
  switch ((p.g.Hn + 1) / 2) {
    LCSA_K1_CASE(1)
    LCSA_K1_CASE(2)
    LCSA_K1_CASE(3)
    LCSA_K1_CASE(4)
    LCSA_K1_CASE(5)
    LCSA_K1_CASE(6)
    LCSA_K1_CASE(7)
    LCSA_K1_CASE(8)
    default: return cudaErrorInvalidValue;
  }
#undef LCSA_K1_CASE
}

}  // namespace lcsa
