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
// never depends on timing. The sort key is (order-preserving score bits << 32)
// | (~candidate number); candidates run in ascending block order, so one
// descending sort of unique keys gives the k best with ties broken toward the
// lower block index. The CSR row offsets depend only on
// the geometry and are computed once when the plan is made.
#include "lcsa_internal.h"

namespace lcsa {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kCandPerIter = 4;  // candidates in flight per warp
constexpr int kRankMax = 512;    // admissible sets up to this size: rank selection, else bitonic sort

__device__ __forceinline__ unsigned order_bits(float s) {
  const unsigned u = __float_as_uint(s + 0.0f);  // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

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
  auto cand_block = [&](int c) {
    const int tk = fdiv(c, m_per), r2 = c - tk * per;
    const int hr = fdiv(r2, m_nw), wr = r2 - hr * nw;
    return tk * g.bpf + (h0 + hr) * g.nWb + (w0 + wr);
  };

  const float4 qv = reinterpret_cast<const float4*>(p.pooled_q + int64_t(rr) * kHeadDim)[lane];
  const float4* pk = reinterpret_cast<const float4*>(p.pooled_k + int64_t(bh) * g.nKB * kHeadDim);

  if (blockIdx.x == 0)
    for (int c = threadIdx.x; c < p.n_clear; c += kThreads) p.clear_cnt[c] = 0u;
  for (int c = threadIdx.x; c < p.sort_n; c += kThreads) {
    flag[c] = 0;
    if (c >= nc) keys[c] = 0ull;  // padding sorts last
  }
  // Sort key: (order-preserving score bits << 32) | ~c, so equal scores go to
  // the lower candidate, i.e. the lower block index.
  for (int c0 = warp * kCandPerIter; c0 < nc; c0 += kWarps * kCandPerIter) {
    float4 kv[kCandPerIter];
#pragma unroll
    for (int u = 0; u < kCandPerIter; ++u) {
      const int c = c0 + u;
      kv[u] = c < nc ? pk[int64_t(cand_block(c)) * (kHeadDim / 4) + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
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
  if (nc <= kRankMax) {
    // rank selection: candidate c is kept when fewer than k keys beat it (keys
    // are unique); every thread reads the same key at each step (broadcast)
    for (int c = threadIdx.x; c < nc; c += kThreads) {
      const unsigned long long mine = keys[c];
      int above = 0;
      int j = 0;
      for (; j + 1 < nc; j += 2) {
        const ulonglong2 kk = *reinterpret_cast<const ulonglong2*>(keys + j);
        above += (kk.x > mine) + (kk.y > mine);
      }
      if (j < nc) above += keys[j] > mine;
      flag[c] = above < keff;
    }
  } else {
    // bitonic sort, descending, then mark the first k
    const int n = p.sort_n;
    for (int k = 2; k <= n; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = threadIdx.x; i < n; i += kThreads) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const unsigned long long a = keys[i], bk = keys[ixj];
            const bool desc = (i & k) == 0;
            if (desc ? (a < bk) : (a > bk)) {
              keys[i] = bk;
              keys[ixj] = a;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int i = threadIdx.x; i < keff; i += kThreads) flag[0xFFFFFFFFu - unsigned(keys[i] & 0xFFFFFFFFull)] = 1;
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
  int pos = p.row_ptr[rr] + base + incl - cnt;
  for (int c = c_beg; c < c_end; ++c) {
    if (flag[c]) p.col_idx[pos++] = cand_block(c);
  }
}

}  // namespace

size_t select_smem_bytes(int sort_n) { return size_t(sort_n) * (sizeof(unsigned long long) + 1); }

cudaError_t launch_select(const K2Params& p, cudaStream_t s) {
  const size_t smem = select_smem_bytes(p.sort_n);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  const int rows = p.g.B * p.g.Hn * p.g.nQB;
  select_kernel<<<rows, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace lcsa
