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
// Work split: a persistent grid of one CTA per SM (8 compute warps and one
// copy warp); CTA c owns a contiguous range of the combined row list (query
// blocks, then key blocks; a block is bt * bh rows of bw tokens). Each row is
// one contiguous run of bw * heads * head_dim bf16 in the raster input, so the
// copy warp streams the rows into a ring of shared-memory stages with bulk
// asynchronous copies (cp.async.bulk, completion counted on a "full"
// mbarrier per stage) several rows ahead. Warp w takes tokens w, w+8, ... of
// a row, lane l the 16-byte chunks l, l+32, ... of a token (conflict-free
// shared loads), so each lane always holds the same channels and its pooled
// sums live in registers (gains: a lane-contiguous table in shared memory).
// The sum of squares is a warp-shuffle reduction. Each lane writes its
// results back over the chunks it read, so a finished stage holds the row's
// q^ / k^ in raster order; each compute warp then arrives on the stage's
// "done" mbarrier and goes on to the next row without waiting for the
// others. Once all have arrived, the copy warp writes the stage out with one
// bulk tensor store (a box of all heads x bw tokens over the head-major
// layout) and refills it when the store has read it. Pooled sums are added in
// a fixed order: per lane over its tokens, then over the warps (at the end of
// each block's rows, the only point where the compute warps synchronise),
// and for a block cut between two CTAs, first part plus second part; so the
// pooled values, and hence the block selection, do not depend on timing.
#include "lcsa_internal.h"

namespace lcsa {
namespace {

constexpr int kRedRows = 2;  // rows of the pooled-sum reduction buffer

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

// bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 word, so
// unpacking is integer shifts and masks, which leaves the conversion unit free.
// The bf16 words become float pairs for packed fp32x2 arithmetic: e[qg]
// holds elements (4qg, 4qg+2), o[qg] elements (4qg+1, 4qg+3), i.e. the first
// and second members of the rotation pairs 2qg and 2qg+1.
__device__ __forceinline__ void unpack_eo(const uint4& r, float2 (&e)[2], float2 (&o)[2]) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int qg = 0; qg < 2; ++qg) {
    e[qg] = make_float2(__uint_as_float(w[2 * qg] << 16), __uint_as_float(w[2 * qg + 1] << 16));
    o[qg] = make_float2(__uint_as_float(w[2 * qg] & 0xFFFF0000u), __uint_as_float(w[2 * qg + 1] & 0xFFFF0000u));
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

constexpr int kMaxStages = 8;  // 128 bytes of mbarriers: full[8], done[8]
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

// Block number bid of the combined list (the processed query blocks, then the
// key blocks of the k input) -> tensor, batch element, output block, the
// input frame and the KV-window frame of its first token.
struct BlockRef {
  bool is_q;
  int b, blk, nblk, t_in0, t_win0, y0, x0;
};
__device__ __forceinline__ BlockRef block_ref(const K1Params& p, int bid) {
  const Grid& g = p.g;
  BlockRef r;
  r.is_q = bid < p.n_qblk;
  int rem;
  if (r.is_q) {
    r.nblk = g.nQB;
    r.b = bid / g.nQB;
    r.blk = bid % g.nQB;
    const int tb = r.blk / g.bpf;
    rem = r.blk % g.bpf;
    r.t_in0 = tb * g.bt;
    r.t_win0 = r.t_in0 + (g.Tkv - g.Tq);  // query frames close the KV window
  } else {
    const int bg = bid - p.n_qblk, per_b = p.k_in_fb * g.bpf;
    r.nblk = g.nKB;
    r.b = bg / per_b;
    const int bi = bg % per_b, tb = bi / g.bpf;
    rem = bi % g.bpf;
    const int wfb = p.k_first_fb + tb;
    r.t_in0 = tb * g.bt;
    r.t_win0 = wfb * g.bt;
    r.blk = ((p.slot0_fb + wfb) % p.ring_fb) * g.bpf + rem;
  }
  r.y0 = (rem / g.nWb) * g.bh;
  r.x0 = (rem % g.nWb) * g.bw;
  return r;
}

// D = head_dim (64 or 128); CPL = 16-byte chunks per lane per token =
// ceil(heads * D / 8 / 32); FULL: every lane's CPL chunks exist; HEAD:
// per-head norm scope.
// Warps per CTA. (16, one token of a 16-token row each, measured slower: a
// lane's pooled sums and token do not fit 128 registers without spills.)
template <int CPL>
__host__ __device__ constexpr int k1_warps() { return 8; }

// A processed row (bw tokens x heads x head_dim, token-major as it arrived)
// goes from its ring stage to q^ / k^ in one bulk tensor store: the map's box
// is (head_dim channels, all heads, bw tokens of one block) over the head-major
// layout, so the shared-memory side is exactly the raster row.
__device__ __forceinline__ void store_row(const CUtensorMap* map, uint32_t src, int r_tok, int blk, int b) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4, %5}], [%6];" ::"l"(map), "r"(0),
      "r"(0), "r"(r_tok), "r"(blk), "r"(b), "r"(src)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Barrier of the compute warps only (named barrier 1; the copy warp never
// joins it), plain and with an AND over the threads' votes.
__device__ __forceinline__ void compute_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}
__device__ __forceinline__ bool compute_sync_and(int nthreads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(uint32_t(v)), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void record_timeout(unsigned* err, unsigned site) {
  if (atomicCAS(err, kDevErrNone, kDevErrTimeout) == kDevErrNone) {
    err[1] = site;
    err[2] = blockIdx.x;
  }
}

// Warps 0..NW-1 compute; warp NW is the copy warp (one lane issues every bulk
// copy, so the compute warps never block on the copy engine).
template <int D, int CPL, bool FULL, bool HEAD>
__global__ void __launch_bounds__((k1_warps<CPL>() + 1) * 32, 1)
    prologue_kernel(const __grid_constant__ CUtensorMap tm_qhat, const __grid_constant__ CUtensorMap tm_khat,
                    const K1Params p, int stages, uint32_t row_bytes) {
  constexpr int NW = k1_warps<CPL>(), NT = NW * 32;
  extern __shared__ __align__(128) uint8_t smem[];
  const Grid& g = p.g;
  const uint32_t bars = smem_u32(smem);
  // ring stages start on a 128-byte boundary (bulk tensor copies need it)
  uint8_t* ring = smem + kBarBytes + (128u - (bars + kBarBytes) % 128u) % 128u;
  float* red = reinterpret_cast<float*>(ring + size_t(stages) * row_bytes);  // [kRedRows][C]
  // gains of q and k, [tensor][c4][half][lane] float4: lane-contiguous, so conflict-free
  float4* gsm = reinterpret_cast<float4*>(red + kRedRows * g.C);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunks = g.C / 8;
  const int R = g.bt * g.bh;  // rows per block
  const int total = p.n_qblk + g.B * p.k_in_fb * g.bpf;
  // this CTA's rows: a contiguous range of the combined row list (blocks in
  // order, rows of a block in order); every range holds at least R rows, so a
  // block is cut by at most one range boundary
  const int64_t nrows = int64_t(total) * R;
  const int64_t lo = nrows * blockIdx.x / gridDim.x, hi = nrows * (blockIdx.x + 1) / gridDim.x;
  const int my_rows = int(hi - lo);
  // RoPE pairs on the frame / row / column axes of a head: (22, 21, 21) for
  // head_dim 128, (12, 10, 10) for 64
  constexpr int PH = D / 6, PT = D / 2 - 2 * PH;

  // full[s]: the stage's row has landed; done[s]: every compute warp has
  // finished the stage's row in place
  auto full_bar = [&](int st) { return bars + 8u * uint32_t(st); };
  auto done_bar = [&](int st) { return bars + 8u * uint32_t(kMaxStages + st); };

  // Order of the range's rows: the cut segments first (the head [lo, a),
  // the tail [bb, hi)), then the complete blocks [a, bb). The partial sums of
  // the cut blocks are then merged early, while the ring streams later rows,
  // and the range ends with a complete block, which needs no merge. (a <= bb:
  // the range holds at least R rows, so it reaches a block boundary.)
  const int64_t a = (lo + R - 1) / R * R, bb = hi / R * R;
  const int nh = int(a - lo), nt = int(hi - bb);
  auto grow_of = [&](int k) -> int64_t {
    return k < nh ? lo + k : (k < nh + nt ? bb + (k - nh) : a + (k - nh - nt));
  };

  // source of the CTA's row number k
  auto row_src = [&](int k) -> const void* {
    const int64_t grow = grow_of(k);
    const BlockRef br = block_ref(p, int(grow / R));
    const int r = int(grow % R);
    const int64_t tok = (int64_t(br.t_in0 + r / g.bh) * g.gh + br.y0 + r % g.bh) * g.gw + br.x0;
    const __nv_bfloat16* x = br.is_q ? p.q : p.k;
    const int64_t L = br.is_q ? g.Lq : p.Lk_in;
    return x + (int64_t(br.b) * L + tok) * g.C;
  };
  auto issue = [&](int gi) {
    const int s = gi % stages;
    bulk_row(smem_u32(ring + size_t(s) * row_bytes), row_src(gi), row_bytes, full_bar(s));
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full_bar(s)));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(done_bar(s)), "r"(NW));
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == NW) {
    // copy warp: rows in as far ahead as the ring allows; each finished row
    // out with one bulk tensor store, its stage refilled once the store has
    // read it
    if (lane == 0) {
      int issued = min(stages, my_rows);
      for (int k = 0; k < issued; ++k) issue(k);
      bool cok = true;
      for (int k = 0; k < my_rows; ++k) {
        const int s = k % stages;
        if (!(cok = mbar_wait_bounded(done_bar(s), uint32_t(k / stages) & 1u))) break;
        const int64_t grow = grow_of(k);
        const BlockRef br = block_ref(p, int(grow / R));
        store_row(br.is_q ? &tm_qhat : &tm_khat, smem_u32(ring + size_t(s) * row_bytes), int(grow % R) * g.bw,
                  br.blk, br.b);
        if (k + stages < my_rows) {
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          issue(k + stages);
          issued = k + stages + 1;
        }
      }
      // stores finish before the CTA exits
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
      if (!cok) {
        // the compute warps stopped: record it, then give the loads still in
        // flight a bounded chance to land before shared memory goes away
        record_timeout(p.err, 2);
        for (int k = max(0, issued - stages); k < issued; ++k)
          (void)mbar_wait_bounded(full_bar(k % stages), uint32_t(k / stages) & 1u);
      }
    }
    return;
  }

  // the gains table (compute warps; the first rows are already on their way)
  for (int idx = threadIdx.x; idx < 2 * CPL * 64; idx += NT) {
    const int rem = idx % (CPL * 64);
    const int c = (rem / 64) * 32 + rem % 32, half = (rem / 32) % 2;
    const float* gamma = idx < CPL * 64 ? p.gamma_q : p.gamma_k;
    gsm[idx] = c < nchunks ? __ldg(reinterpret_cast<const float4*>(gamma + c * 8 + half * 4))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  compute_sync(NT);

  constexpr int kChunksPerHead = D / 8;
  const int jb = 4 * (lane & (kChunksPerHead - 1));  // first RoPE pair of this lane (same in every head)
  float2 ae[CPL][2], ao[CPL][2];  // pooled sums, e / o layout of unpack_eo
  __shared__ int combine;
  int gi = 0;  // rows of this CTA consumed so far
  bool ok = true;
  while (gi < my_rows && ok) {
    // one segment: the rows [r_begin, r_end) of block bid that this CTA owns
    const int64_t g0 = grow_of(gi);
    const int bid = int(g0 / R);
    const int r_begin = int(g0 % R);
    const int r_end = gi < nh ? R : (gi < nh + nt ? nt : R);
    const BlockRef br = block_ref(p, bid);
    const float4* gtab = gsm + (br.is_q ? 0 : CPL * 64);
    float* pooled = br.is_q ? p.pooled_q : p.pooled_k;
#pragma unroll
    for (int c4 = 0; c4 < CPL; ++c4)
#pragma unroll
      for (int qg = 0; qg < 2; ++qg) ae[c4][qg] = ao[c4][qg] = make_float2(0.f, 0.f);
    for (int r = r_begin; r < r_end; ++r, ++gi) {
      const int s = gi % stages;
      // after a failed wait the warp skips to the segment's end, where the
      // compute warps agree on it
      if (!ok || !(ok = __all_sync(0xffffffffu, mbar_wait_bounded(full_bar(s), uint32_t(gi / stages) & 1u))))
        continue;
      const int t = br.t_win0 + r / g.bh, y = br.y0 + r % g.bh;  // t: KV-window frame
      uint4* row = reinterpret_cast<uint4*>(ring + size_t(s) * row_bytes);
      // head-sharded layer: the row's per-token sums of squares over all heads
      const float* ss_row =
          (!HEAD && p.ss_ext) ? p.ss_ext + (br.is_q ? int64_t(br.b) * g.Lq : int64_t(g.B) * g.Lq + int64_t(br.b) * p.Lk_in) +
                         (int64_t(br.t_in0 + r / g.bh) * g.gh + y) * g.gw + br.x0
                   : nullptr;
      for (int i = warp; i < g.bw; i += NW) {
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
          const int idx = j < PT        ? t * PT + j
                          : j < PT + PH ? p.rope_h_off + y * PH + (j - PT)
                                        : p.rope_w_off + xc * (D / 2 - PT - PH) + (j - PT - PH);
          cs[qd] = __ldg(p.rope + idx);
        }
        // RMSNorm scale(s), folded into the rotation: x^ = rot(rs * (x * gamma)).
        // ca/cb/nb[qg] = rs * (cos, sin, -sin) of the pairs 2qg and 2qg+1 (per
        // token; with the head scope, per chunk inside the chunk loop).
        float2 ca[2], cb[2], nb[2];
        float rr_h[HEAD ? CPL : 1];
        auto coefs = [&](float rr) {
#pragma unroll
          for (int qg = 0; qg < 2; ++qg) {
            const float2 cosv = make_float2(cs[2 * qg].x, cs[2 * qg + 1].x);
            const float2 sinv = make_float2(cs[2 * qg].y, cs[2 * qg + 1].y);
            ca[qg] = __fmul2_rn(make_float2(rr, rr), cosv);
            cb[qg] = __fmul2_rn(make_float2(rr, rr), sinv);
            nb[qg] = __fmul2_rn(make_float2(-rr, -rr), sinv);
          }
        };
        if (!HEAD) {
          // the order of sumsq_kernel's sums (an accumulator per qg, then the
          // butterfly), so a one-rank sharded call equals the plain call
          float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int c4 = 0; c4 < CPL; ++c4) {
            float2 e[2], o[2];
            unpack_eo(raw[c4], e, o);
#pragma unroll
            for (int qg = 0; qg < 2; ++qg) {
              acc[qg] = __ffma2_rn(e[qg], e[qg], acc[qg]);
              acc[qg] = __ffma2_rn(o[qg], o[qg], acc[qg]);
            }
          }
          float ss = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          if (ss_row) ss = __ldg(ss_row + i);  // head-sharded layer: the sum over all its heads
          coefs(rsqrtf(ss * p.norm_inv_c + p.eps));
        } else {
#pragma unroll
          for (int c4 = 0; c4 < (HEAD ? CPL : 1); ++c4) {
            float2 e[2], o[2];
            unpack_eo(raw[c4], e, o);
            float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int qg = 0; qg < 2; ++qg) {
              ss2 = __ffma2_rn(e[qg], e[qg], ss2);
              ss2 = __ffma2_rn(o[qg], o[qg], ss2);
            }
            float ss = ss2.x + ss2.y;
#pragma unroll
            // the lanes of one head: 16 (head_dim 128) or 8 (64)
            for (int o2 = kChunksPerHead / 2; o2 > 0; o2 >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o2);
            rr_h[c4] = rsqrtf(ss * (1.0f / float(D)) + p.eps);
          }
        }
#pragma unroll
        for (int c4 = 0; c4 < CPL; ++c4) {
          const int c = c4 * 32 + lane;
          if (!FULL && c >= nchunks) continue;
          if (HEAD) coefs(rr_h[HEAD ? c4 : 0]);
          float2 e[2], o[2];
          unpack_eo(raw[c4], e, o);
          const float4 g0 = gtab[(c4 * 2) * 32 + lane], g1 = gtab[(c4 * 2 + 1) * 32 + lane];
          const float2 ge[2] = {make_float2(g0.x, g0.z), make_float2(g1.x, g1.z)};
          const float2 go[2] = {make_float2(g0.y, g0.w), make_float2(g1.y, g1.w)};
          uint32_t w[4];
#pragma unroll
          for (int qg = 0; qg < 2; ++qg) {
            const float2 ue = __fmul2_rn(e[qg], ge[qg]), uo = __fmul2_rn(o[qg], go[qg]);
            const float2 oe = __ffma2_rn(uo, nb[qg], __fmul2_rn(ue, ca[qg]));  // first members
            const float2 oo = __ffma2_rn(uo, ca[qg], __fmul2_rn(ue, cb[qg]));  // second members
            ae[c4][qg] = __fadd2_rn(ae[c4][qg], oe);
            ao[c4][qg] = __fadd2_rn(ao[c4][qg], oo);
            w[2 * qg] = pack2(oe.x, oo.x);
            w[2 * qg + 1] = pack2(oe.y, oo.y);
          }
          row[i * nchunks + c] = make_uint4(w[0], w[1], w[2], w[3]);  // in place: this lane read it
        }
      }
      // the row's results, written in place, become visible to the bulk copy
      // engine; this warp is done with stage s
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(done_bar(s)) : "memory");
    }
    if (!compute_sync_and(NT, ok)) {
      ok = false;
      break;
    }
    // warp partials -> segment sum: with 16 warps, warp w + 8 first leaves its
    // sums in row w and warp w adds its own; then the 8 rows are added in order
    float* mine = red + (warp % kRedRows) * g.C;
#pragma unroll
    for (int round = 0; round < NW / kRedRows; ++round) {
      if (warp / kRedRows == NW / kRedRows - 1 - round) {
#pragma unroll
        for (int c4 = 0; c4 < CPL; ++c4) {
          const int c = c4 * 32 + lane;
          if (FULL || c < nchunks) {
#pragma unroll
            for (int qg = 0; qg < 2; ++qg) {
              float4* slot = reinterpret_cast<float4*>(mine + c * 8) + qg;
              float4 v = make_float4(ae[c4][qg].x, ao[c4][qg].x, ae[c4][qg].y, ao[c4][qg].y);
              if (round > 0) {
                const float4 prev = *slot;
                v.x += prev.x; v.y += prev.y; v.z += prev.z; v.w += prev.w;
              }
              *slot = v;
            }
          }
        }
      }
      compute_sync(NT);
    }
    const float inv_nb = 1.0f / float(g.nb);
    float* pooled_row = pooled + (int64_t(br.b) * g.Hn * br.nblk + br.blk) * D;  // + head * nblk * d + dd
    const int64_t head_stride = int64_t(br.nblk) * D;
    auto warp_sum = [&](int e) {
      float sum = red[e];
#pragma unroll
      for (int w = 1; w < kRedRows; ++w) sum += red[w * g.C + e];
      return sum;
    };
    if (r_begin == 0 && r_end == R) {
      for (int e = threadIdx.x; e < g.C; e += NT)
        pooled_row[(e / D) * head_stride + e % D] = warp_sum(e) * inv_nb;
    } else {
      // A block cut between CTA c and c + 1: CTA c holds its first rows (part
      // 0), CTA c + 1 the rest (part 1). Each writes its part to the cut's
      // slot; the second to arrive adds part 0 + part 1 (always in that
      // order) and writes the mean.
      const int cut = r_begin == 0 ? int(blockIdx.x) : int(blockIdx.x) - 1;
      float* part = p.split_part + size_t(cut) * 2 * g.C;
      float* mypart = part + (r_begin == 0 ? 0 : g.C);
      for (int e = threadIdx.x; e < g.C; e += NT) mypart[e] = warp_sum(e);
      // The barrier orders the CTA's part before thread 0's count, whose
      // release publishes it at GPU scope and whose acquire (for the second
      // arrival) makes the other part visible; the barrier after it extends
      // that to every thread.
      compute_sync(NT);
      if (threadIdx.x == 0) {
        unsigned old;
        asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(old) : "l"(p.split_cnt + cut) : "memory");
        combine = old == 1u;
      }
      compute_sync(NT);
      if (combine) {
        for (int e = threadIdx.x; e < g.C; e += NT)
          pooled_row[(e / D) * head_stride + e % D] =
              (__ldcg(part + e) + __ldcg(part + g.C + e)) * inv_nb;
      }
    }
    compute_sync(NT);  // red and combine are rewritten by the next segment
  }
  // a row never arrived (the copy warp then waits out the loads in flight)
  if (!ok && threadIdx.x == 0) record_timeout(p.err, 1);
}

template <int D, int CPL, bool FULL, bool HEAD>
cudaError_t launch_cpl(const K1Params& p, cudaStream_t s) {
  const int nblocks = p.n_qblk + p.g.B * p.k_in_fb * p.g.bpf;
  if (nblocks <= 0) return cudaSuccess;
  const uint32_t row_bytes = uint32_t(p.g.bw) * uint32_t(p.g.C) * 2u;
  const uint32_t red_bytes = uint32_t(kRedRows) * uint32_t(p.g.C) * 4u + 2u * CPL * 64u * 16u;  // + gains
  int stages = int((kSmemBudget - kBarBytes - 128 - red_bytes) / row_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2 || p.num_sms <= 0) return cudaErrorInvalidValue;
  const size_t smem = kBarBytes + 128 + size_t(stages) * row_bytes + red_bytes;  // + alignment of the ring
  cudaError_t e =
      cudaFuncSetAttribute(prologue_kernel<D, CPL, FULL, HEAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  int grid = nblocks < p.num_sms ? nblocks : p.num_sms;
  if (grid > kMaxK1Ctas) grid = kMaxK1Ctas;
  CUtensorMap tm_qhat, tm_khat;
  if ((e = make_xhat_row_map(&tm_qhat, p.qhat, p.g, p.g.nQB)) != cudaSuccess ||
      (e = make_xhat_row_map(&tm_khat, p.khat, p.g, p.g.nKB)) != cudaSuccess)
    return e;
  prologue_kernel<D, CPL, FULL, HEAD><<<grid, (k1_warps<CPL>() + 1) * 32, smem, s>>>(tm_qhat, tm_khat, p, stages,
                                                                                    row_bytes);
  return cudaGetLastError();
}

// One warp per token (q tokens, then k tokens): every 16-byte chunk of the
// token is requested before any is summed (at most 8 per lane: heads <= 16),
// fp32 squares, then a butterfly; the same order of additions as the
// prologue's own sums of squares.
__global__ void __launch_bounds__(256) sumsq_kernel(const __nv_bfloat16* xq, int64_t nq, const __nv_bfloat16* xk,
                                                    int64_t nk, int channels, float* ss) {
  const int64_t t = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= nq + nk) return;
  const uint4* row = reinterpret_cast<const uint4*>(t < nq ? xq + t * channels : xk + (t - nq) * channels);
  const int nch = channels / 8;
  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = lane + 32 * i;
    v[i] = c < nch ? __ldg(row + c) : make_uint4(0u, 0u, 0u, 0u);
  }
  float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float2 e[2], o[2];
    unpack_eo(v[i], e, o);
#pragma unroll
    for (int qg = 0; qg < 2; ++qg) {
      acc[qg] = __ffma2_rn(e[qg], e[qg], acc[qg]);
      acc[qg] = __ffma2_rn(o[qg], o[qg], acc[qg]);
    }
  }
  float sum = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
#pragma unroll
  for (int o2 = 16; o2 > 0; o2 >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o2);
  if (lane == 0) ss[t] = sum;
}

}  // namespace

cudaError_t launch_rope_table(float2* table, int Tkv, int gh, int gw, int t0, int d, cudaStream_t s) {
  const RopeSplit rs = rope_split(d);
  const int n = Tkv * rs.pairs_t + gh * rs.pairs_h + gw * rs.pairs_w;
  rope_table_kernel<<<(n + 255) / 256, 256, 0, s>>>(table, Tkv, gh, gw, t0, rs);
  return cudaGetLastError();
}

cudaError_t launch_sumsq(const __nv_bfloat16* q, int64_t nq, const __nv_bfloat16* k, int64_t nk, int channels,
                         float* ss, cudaStream_t s) {
  if (channels % 8 || channels > 2048) return cudaErrorInvalidValue;
  if (nq + nk <= 0) return cudaSuccess;
  sumsq_kernel<<<unsigned((nq + nk + 7) / 8), 256, 0, s>>>(q, nq, k, nk, channels, ss);
  return cudaGetLastError();
}

cudaError_t launch_prologue(const K1Params& p, cudaStream_t s) {
  const int nchunks = p.g.C / 8;
  const bool full = nchunks % 32 == 0, head = p.norm_scope != 0;
#define LCSA_K1_CASE(d, n)                                                                          \
  case n:                                                                                           \
    if (full) return head ? launch_cpl<d, n, true, true>(p, s) : launch_cpl<d, n, true, false>(p, s); \
    return head ? launch_cpl<d, n, false, true>(p, s) : launch_cpl<d, n, false, false>(p, s);
  if (p.g.D == 128) {
    switch ((nchunks + 31) / 32) {
      LCSA_K1_CASE(128, 1)
      LCSA_K1_CASE(128, 2)
      LCSA_K1_CASE(128, 3)
      LCSA_K1_CASE(128, 4)
      LCSA_K1_CASE(128, 5)
      LCSA_K1_CASE(128, 6)
      LCSA_K1_CASE(128, 7)
      LCSA_K1_CASE(128, 8)
      default: return cudaErrorInvalidValue;
    }
  }
  if (p.g.D == 64) {
    switch ((nchunks + 31) / 32) {
      LCSA_K1_CASE(64, 1)
      LCSA_K1_CASE(64, 2)
      LCSA_K1_CASE(64, 3)
      LCSA_K1_CASE(64, 4)
      default: return cudaErrorInvalidValue;
    }
  }
  return cudaErrorInvalidValue;
#undef LCSA_K1_CASE
}

}  // namespace lcsa
