// K2: LCSA block selection. For every (batch, head, query block) row: score
// each KV block inside the local window by the dot product of the pooled q
// and pooled k vectors, keep the k best (equal scores: lower block index
// first) and write the kept block indices in ascending order into the row's
// CSR slot.
//
// Pages: "FlashVSR: From 17.2 FPS to 57.3 FPS at 768x1408", What Was Actually
// Slow (mask selection as glue) and Rebuild sparse attention for Hopper (fused
// CSR construction); "FlashVSR Inference" skill, Non-Negotiable Streaming
// Contract (local_range, topk_ratio); "FlashVSR - Real-Time Diffusion-Based
// Video Super-Resolution", How it works (attention limited to local patches).
//
// Determinism: a score is the fp32 sum of four products per lane followed by
// a butterfly over the warp; every lane ends with the same bits, and the order
// never depends on timing. Each candidate's key is (order-preserving score
// bits << 32) | ~candidate number; candidates run in ascending block order, so
// the k largest keys are the k best blocks with equal scores going to the
// lower block index. A radix selection finds the k-th largest score in four
// 8-bit digits (one shared histogram each) and a block scan takes the
// lowest-numbered candidates among those equal to it (measured faster than
// both a bitonic sort and counting each candidate's rank, at 180 and at up
// to 726 candidates per row). The CSR row offsets
// depend only on the geometry and are computed once when the plan is made.
//
// Threshold reuse (the same pages, Remove the remaining control-plane tax and
// Measured Results: the mask-generation threshold of the previous steady
// chunk reused per DiT block): a selecting call records each row's k-th best
// score (its order bits); a reuse call keeps every admissible block scoring at
// least that, in ascending order, into the row's slot of a padded CSR with a
// count per row; a row where no block reaches it keeps its best block.
#include "lcsa_internal.h"

namespace lcsa {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kCandPerIter = 4;  // candidates in flight per warp

__device__ __forceinline__ unsigned order_bits(float s) {
  const unsigned u = __float_as_uint(s + 0.0f);  // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// D: head_dim (64 or 128); the first D / 4 lanes hold a pooled vector's
// float4s, the others add zeros.
template <int D>
__global__ void __launch_bounds__(kThreads) select_kernel(const K2Params p) {
  extern __shared__ __align__(16) unsigned long long keys[];  // [sort_n], then flags [sort_n] bytes
  unsigned char* flag = reinterpret_cast<unsigned char*>(keys + p.sort_n);
  __shared__ int warp_sum[kWarps];
  const Grid& g = p.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr = blockIdx.x;
  const int bh = rr / g.nQB, qb = rr % g.nQB;
  const int rem = qb % g.bpf, hb = rem / g.nWb, wb = rem % g.nWb;
  int h0 = 0, h1 = g.nHb - 1, w0 = 0, w1 = g.nWb - 1;
  if (p.radius >= 0) {
    h0 = max(hb - p.radius, 0);
    h1 = min(hb + p.radius, g.nHb - 1);
    w0 = max(wb - p.radius, 0);
    w1 = min(wb + p.radius, g.nWb - 1);
  }
  const int nh = h1 - h0 + 1, nw = w1 - w0 + 1, per = nh * nw;
  const int nc = (g.nKB / g.bpf) * per;  // admissible blocks, ascending index order

  // Candidate c (ascending block order) -> block index, with exact divisions
  // by the row's constants: floor(c / d) = (c * ceil(2^32 / d)) >> 32 while
  // c * d < 2^32 (here both are below 2^13).
  auto magic = [](int d) { return 0xFFFFFFFFull / unsigned(d) + 1ull; };
  auto fdiv = [](int c, unsigned long long m) { return int((unsigned long long)unsigned(c) * m >> 32); };
  const unsigned long long m_per = magic(per), m_nw = magic(nw);
  auto cand_block = [&](int c, bool ring) {
    const int tk = fdiv(c, m_per), r2 = c - tk * per;
    const int hr = fdiv(r2, m_nw), wr = r2 - hr * nw;
    int slot = tk;  // where its pooled k is stored: ring slot (slot0 + tk) mod ring, both below ring
    if (ring) {
      slot += p.slot0_fb;
      if (slot >= p.ring_fb) slot -= p.ring_fb;
    }
    return slot * g.bpf + (h0 + hr) * g.nWb + (w0 + wr);
  };

  constexpr int kLanes = D / 4;  // lanes that hold part of a pooled vector
  const float4 qv = lane < kLanes ? reinterpret_cast<const float4*>(p.pooled_q + int64_t(rr) * D)[lane]
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
  const float4* pk = reinterpret_cast<const float4*>(p.pooled_k + int64_t(bh) * g.nKB * D);

  if (blockIdx.x == 0)
    for (int c = threadIdx.x; c < p.n_clear; c += kThreads) p.clear_cnt[c] = 0u;
  for (int c = threadIdx.x; c < nc; c += kThreads) flag[c] = 0;
  // Sort key: (order-preserving score bits << 32) | ~c, so equal scores go to
  // the lower candidate, i.e. the lower block index.
  for (int c0 = warp * kCandPerIter; c0 < nc; c0 += kWarps * kCandPerIter) {
    float4 kv[kCandPerIter];
#pragma unroll
    for (int u = 0; u < kCandPerIter; ++u) {
      const int c = c0 + u;
      kv[u] = (c < nc && lane < kLanes) ? pk[int64_t(cand_block(c, true)) * kLanes + lane]
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kCandPerIter; ++u) {
      const int c = c0 + u;
      if (c >= nc) break;  // warp-uniform
      float s = qv.x * kv[u].x;
      s = fmaf(qv.y, kv[u].y, s);
      s = fmaf(qv.z, kv[u].z, s);
      s = fmaf(qv.w, kv[u].w, s);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) keys[c] = ((unsigned long long)order_bits(s) << 32) | (0xFFFFFFFFu - unsigned(c));
    }
  }
  __syncthreads();

  const int keff = min(p.topk, nc);
  if (p.reuse) {
    // threshold reuse: every admissible block scoring at least the recorded
    // k-th best score of this row
    const unsigned th = p.thresh[rr];
    int any = 0;
    for (int c = threadIdx.x; c < nc; c += kThreads) {
      const unsigned char f = unsigned(keys[c] >> 32) >= th;
      flag[c] = f;
      any |= f;
    }
    if (!__syncthreads_or(any)) {
      // no block reaches it: keep the row's best block (largest key: highest
      // score, then the lower block)
      __shared__ unsigned long long wmax[kWarps];
      unsigned long long mk = 0ull;
      for (int c = threadIdx.x; c < nc; c += kThreads) mk = keys[c] > mk ? keys[c] : mk;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long t = __shfl_xor_sync(0xffffffffu, mk, o);
        mk = t > mk ? t : mk;
      }
      if (lane == 0) wmax[warp] = mk;
      __syncthreads();
      if (threadIdx.x == 0) {
        for (int w = 1; w < kWarps; ++w) mk = wmax[w] > mk ? wmax[w] : mk;
        flag[0xFFFFFFFFu - unsigned(mk & 0xFFFFFFFFull)] = 1;
      }
    }
  } else {
    // the k-th largest score (order-preserving bits, four 8-bit digits from
    // the top, one shared histogram per digit), then all candidates above it
    // and the lowest-numbered `remain` of those equal to it (equal scores go
    // to the lower block).
    __shared__ unsigned hist[256];
    __shared__ unsigned sel_digit, sel_rem;
    const int span = (nc + kThreads - 1) / kThreads;
    const int c_beg = min(int(threadIdx.x) * span, nc), c_end = min(c_beg + span, nc);
    unsigned prefix = 0, pmask = 0, remain = unsigned(keff);
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = threadIdx.x; i < 256; i += kThreads) hist[i] = 0u;
      __syncthreads();
      for (int c = c_beg; c < c_end; ++c) {
        const unsigned sb = unsigned(keys[c] >> 32);
        if ((sb & pmask) == prefix) atomicAdd(&hist[(sb >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        // lane l covers digits 255 - 8l down to 248 - 8l; counts from the top
        unsigned h[8], tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          h[i] = hist[255 - 8 * lane - i];
          tot += h[i];
        }
        unsigned incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        unsigned acc = incl - tot;
        if (acc < remain && remain <= incl) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (acc + h[i] >= remain) {
              sel_digit = unsigned(255 - 8 * lane - i);
              sel_rem = remain - acc;
              break;
            }
            acc += h[i];
          }
        }
      }
      __syncthreads();
      prefix |= sel_digit << shift;
      pmask |= 255u << shift;
      remain = sel_rem;
      __syncthreads();  // hist and sel_* are rewritten by the next digit
    }
    // rank of each tie in ascending candidate order: block exclusive scan
    int ties = 0;
    for (int c = c_beg; c < c_end; ++c) ties += unsigned(keys[c] >> 32) == prefix;
    int tincl = ties;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, tincl, o);
      if (lane >= o) tincl += t;
    }
    if (lane == 31) warp_sum[warp] = tincl;
    __syncthreads();
    int tr = tincl - ties;
    for (int w = 0; w < warp; ++w) tr += warp_sum[w];
    for (int c = c_beg; c < c_end; ++c) {
      const unsigned sb = unsigned(keys[c] >> 32);
      unsigned char keep = sb > prefix;
      if (sb == prefix) keep = unsigned(tr++) < remain;
      flag[c] = keep;
    }
    // the threshold a later reuse call applies (all blocks kept: any score)
    if (p.thresh && threadIdx.x == 0) p.thresh[rr] = keff < nc ? prefix : 0u;
  }
  __syncthreads();
  const int span = (nc + kThreads - 1) / kThreads;
  const int c_beg = threadIdx.x * span, c_end = min(c_beg + span, nc);
  int cnt = 0;
  for (int c = c_beg; c < c_end; ++c) cnt += flag[c];
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_sum[w];
  int* dst = p.reuse ? p.col_pad + int64_t(rr) * p.pad_cap : p.col_idx + p.row_ptr[rr];
  int pos = base + incl - cnt;
  for (int c = c_beg; c < c_end; ++c) {
    if (flag[c]) dst[pos++] = cand_block(c, false);  // window order
  }
  if (p.reuse && threadIdx.x == kThreads - 1) p.row_len[rr] = pos;  // the last thread's end is the row's count
}

// Union of the selections of two query blocks, ascending. A byte per KV
// block marks which candidate rows kept it (bit i for r[i]); in a 2 x 2
// group the two CTAs of the group's pairs both mark all four rows, count the
// unions of either split (columns: r0+r2, r1+r3; rows: r0+r1, r2+r3) and so
// take the same decision; then a block scan emits this pair's union, each
// entry marked with which of its two rows kept it (bit 0 the first, bit 1
// the second), and the pair's rows are recorded for K3.
__global__ void __launch_bounds__(kThreads) pair_union_kernel(const PairParams p) {
  extern __shared__ unsigned mark_words[];  // [ceil(nkb / 4)]: byte c of the array is block c's mark
  const unsigned char* mark = reinterpret_cast<const unsigned char*>(mark_words);
  __shared__ int warp_sum[kWarps];
  __shared__ int split_sum[2][kWarps];
  const int pr = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int c = threadIdx.x; c < (p.nkb + 3) / 4; c += kThreads) mark_words[c] = 0u;
  __syncthreads();
  // the attention's merge state of cut pairs starts at zero
  for (int i = pr * kThreads + threadIdx.x; i < p.cut * 8 * (1 + kCutParts); i += p.npairs * kThreads) {
    if (i < p.cut * 8) p.merge_cnt[i] = 0u;
    else p.merge_ready[i - p.cut * 8] = 0u;
  }
  int r[4], slot;
  pair_candidates(p.g, pr, r, slot);
  // the rows' entries all at once: each sets its own bit of the block's byte
#pragma unroll
  for (int side = 0; side < 4; ++side) {
    const int row = r[side];
    if (row >= 0) {
      const int64_t beg = p.row_len ? int64_t(row) * p.pad_cap : int64_t(p.row_ptr[row]);
      const int n = p.row_len ? p.row_len[row] : p.row_ptr[row + 1] - p.row_ptr[row];
      for (int i = threadIdx.x; i < n; i += kThreads) {
        const int c = p.col_idx[beg + i];
        atomicOr(&mark_words[c >> 2], 1u << ((c & 3) * 8 + side));
      }
    }
  }
  __syncthreads();
  const int span = (p.nkb + kThreads - 1) / kThreads;
  const int c_beg = min(int(threadIdx.x) * span, p.nkb), c_end = min(c_beg + span, p.nkb);
  // the pair's two rows as bits of mark[]
  unsigned first = 1u, second = 2u;
  int ra = r[0], rb = r[1];
  if (slot >= 0) {
    int by_cols = 0, by_rows = 0;
    for (int c = c_beg; c < c_end; ++c) {
      const unsigned m = mark[c];
      by_cols += ((m & 5u) != 0) + ((m & 10u) != 0);
      by_rows += ((m & 3u) != 0) + ((m & 12u) != 0);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      by_cols += __shfl_xor_sync(0xffffffffu, by_cols, o);
      by_rows += __shfl_xor_sync(0xffffffffu, by_rows, o);
    }
    if (lane == 0) {
      split_sum[0][warp] = by_cols;
      split_sum[1][warp] = by_rows;
    }
    __syncthreads();
    int tot_cols = 0, tot_rows = 0;
    for (int w = 0; w < kWarps; ++w) {
      tot_cols += split_sum[0][w];
      tot_rows += split_sum[1][w];
    }
    if (tot_rows < tot_cols) {  // left with right
      first = slot ? 4u : 1u;
      second = slot ? 8u : 2u;
      ra = slot ? r[2] : r[0];
      rb = slot ? r[3] : r[1];
    } else {  // top with bottom
      first = slot ? 2u : 1u;
      second = slot ? 8u : 4u;
      ra = slot ? r[1] : r[0];
      rb = slot ? r[3] : r[2];
    }
  }
  int cnt = 0;
  for (int c = c_beg; c < c_end; ++c) cnt += (mark[c] & (first | second)) != 0;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int pos = incl - cnt;
  for (int w = 0; w < warp; ++w) pos += warp_sum[w];
  int* dst = p.pair_col + int64_t(pr) * p.pair_cap;
  for (int c = c_beg; c < c_end; ++c) {
    const unsigned m = mark[c];
    const int two = ((m & first) ? 1 : 0) | ((m & second) ? 2 : 0);
    if (two) dst[pos++] = c | (two << kPairShift);
  }
  if (threadIdx.x == kThreads - 1) {
    p.pair_len[pr] = pos;
    p.pair_rows[pr] = make_int2(ra, rb);
  }
}

}  // namespace

cudaError_t launch_pair_union(const PairParams& p, cudaStream_t s) {
  if (p.npairs <= 0) return cudaSuccess;
  if (p.nkb > 48 * 1024 - 256) return cudaErrorInvalidValue;  // marks + the kernel's static arrays in 48 KB
  pair_union_kernel<<<p.npairs, kThreads, size_t((p.nkb + 3) / 4) * 4, s>>>(p);
  return cudaGetLastError();
}

size_t select_smem_bytes(int sort_n) { return size_t(sort_n) * (sizeof(unsigned long long) + 1); }

namespace {
template <int D>
cudaError_t launch_select_d(const K2Params& p, cudaStream_t s) {
  const size_t smem = select_smem_bytes(p.sort_n);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  const int rows = p.g.B * p.g.Hn * p.g.nQB;
  select_kernel<D><<<rows, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_select(const K2Params& p, cudaStream_t s) {
  if (p.g.D == 128) return launch_select_d<128>(p, s);
  if (p.g.D == 64) return launch_select_d<64>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace lcsa
