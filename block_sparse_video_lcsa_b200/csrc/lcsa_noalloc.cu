// lcsa_forward_noalloc: the LCSA call for callers that cannot allocate device
// memory.
//
// Some host programs may not call cudaMalloc once they are running: a
// real-time video pipeline or a plugin inside a larger application often
// reserves all of its device memory at start-up and forbids allocation
// afterwards, because cudaMalloc/cudaFree can synchronise the whole device
// and stall the decode, encode and render streams that share it, and because
// a late allocation can fail when another allocator already owns the memory.
// Those callers cannot create an lcsa_plan_t (which allocates its workspace).
// This entry point runs the same three kernels with every intermediate placed
// in a file-scope static device array of LCSA_NOALLOC_WORKSPACE_BYTES, which
// each GPU that loads the library holds until the process exits.
//
// The first call on a device looks up the array's device address there
// (cudaGetSymbolAddress with that device current); make that first call
// before any stream capture. All calls share the one array and it keeps the
// last call's contents, so calls that overlap on the GPU (other streams, other
// host threads) race; serialise them. The kernels overwrite every byte they
// read except the error word, which each call clears first.
#include <cmath>
#include <mutex>

#include "lcsa.h"
#include "lcsa_internal.h"
#include "nvtx_range.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_ws[LCSA_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_ws_mutex;
void* g_ws_addr[kMaxDevices] = {};

// Failures are reported by status code only: composing a message string could
// allocate host memory, which this entry point never does.
lcsa_status_t noalloc_fail(lcsa_status_t st, const char* /*why*/) { return st; }

size_t round256(size_t n) { return (n + 255) & ~size_t(255); }

// k_eff of every (b, h, qb) row and the row offsets, from the geometry alone.
__global__ void noalloc_row_ptr_kernel(int* row_ptr, lcsa::Grid g, int radius, int topk) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const int groups = g.nKB / g.bpf;
  int acc = 0;
  const int rows = g.B * g.Hn * g.nQB;
  for (int row = 0; row < rows; ++row) {
    row_ptr[row] = acc;
    const int rem = (row % g.nQB) % g.bpf;
    const int hb = rem / g.nWb, wb = rem % g.nWb;
    int nh = g.nHb, nw = g.nWb;
    if (radius >= 0) {
      nh = min(hb + radius, g.nHb - 1) - max(hb - radius, 0) + 1;
      nw = min(wb + radius, g.nWb - 1) - max(wb - radius, 0) + 1;
    }
    const int a = groups * nh * nw;
    acc += topk < a ? topk : a;
  }
  row_ptr[rows] = acc;
}

// Sizes of one problem, checked without touching the heap.
struct NoallocGeom {
  lcsa::Grid g;
  int radius, topk, max_window;
  int64_t rows, nnz;
};

lcsa_status_t noalloc_resolve(const lcsa_config_t* c, NoallocGeom* out) {
  if (c->batch < 1 || c->heads < 1 || c->head_dim < 1 || c->q_frames < 1 || c->kv_frames < 1 || c->grid_h < 1 ||
      c->grid_w < 1 || c->block_t < 1 || c->block_h < 1 || c->block_w < 1)
    return noalloc_fail(LCSA_ERR_INVALID_ARG, "sizes must be >= 1");
  if (c->local_range < 0 || (c->local_range != LCSA_UNBOUNDED && c->local_range % 2 == 0))
    return noalloc_fail(LCSA_ERR_INVALID_ARG, "local_range must be odd or 0 (unbounded)");
  if (c->topk < 0 || (c->topk == 0 && !(c->sparse_ratio > 0.f && std::isfinite(c->sparse_ratio))))
    return noalloc_fail(LCSA_ERR_INVALID_ARG, "topk < 0, or topk = 0 without a finite sparse_ratio > 0");
  if ((c->norm_scope != LCSA_NORM_TOKEN && c->norm_scope != LCSA_NORM_HEAD) || !(c->rms_eps > 0.f) ||
      !std::isfinite(c->rms_eps) ||
      !(c->softmax_scale >= 0.f) || !std::isfinite(c->softmax_scale) || c->kv_frame_offset < 0)
    return noalloc_fail(LCSA_ERR_INVALID_ARG, "norm_scope, rms_eps, softmax_scale or kv_frame_offset out of range");
  if (c->kv_frames < c->q_frames || c->grid_h % c->block_h || c->grid_w % c->block_w || c->q_frames % c->block_t ||
      c->kv_frames % c->block_t)
    return noalloc_fail(LCSA_ERR_SHAPE, "kv_frames < q_frames, or the token grid is not divisible by the block");
  const int nb = c->block_t * c->block_h * c->block_w;
  if (c->head_dim != lcsa::kHeadDim || c->heads > lcsa::kMaxHeads || (nb != 64 && nb != 128) ||
      c->block_t * c->block_h > 8)
    return noalloc_fail(LCSA_ERR_UNSUPPORTED, "head_dim, heads or block shape outside what the kernels implement");
  // sizes bounded in floating point before any integer product (2^40
  // elements per tensor at most: every block count below fits an int)
  if (double(c->batch) * double(c->kv_frames) * double(c->grid_h) * double(c->grid_w) * double(c->heads) *
          double(c->head_dim) > double(int64_t(1) << 40))
    return noalloc_fail(LCSA_ERR_UNSUPPORTED, "tensor of more than 2^40 elements");
  lcsa::Grid& g = out->g;
  g.B = c->batch;
  g.Hn = c->heads;
  g.Tq = c->q_frames;
  g.Tkv = c->kv_frames;
  g.gh = c->grid_h;
  g.gw = c->grid_w;
  g.bt = c->block_t;
  g.bh = c->block_h;
  g.bw = c->block_w;
  g.nb = nb;
  g.nHb = c->grid_h / c->block_h;
  g.nWb = c->grid_w / c->block_w;
  g.bpf = g.nHb * g.nWb;
  g.nQB = (c->q_frames / c->block_t) * g.bpf;
  g.nKB = (c->kv_frames / c->block_t) * g.bpf;
  g.Lq = int64_t(c->q_frames) * c->grid_h * c->grid_w;
  g.Lkv = int64_t(c->kv_frames) * c->grid_h * c->grid_w;
  g.C = c->heads * c->head_dim;
  // budget: topk_ratio = sparse_ratio*768*1280/(H*W), H = 16 grid_h, W = 16 grid_w,
  // times the blocks of one latent frame
  int topk = c->topk;
  if (topk == 0) {
    const double k = std::floor(double(c->sparse_ratio) * 983040.0 * double(g.bpf) /
                                ((16.0 * c->grid_h) * (16.0 * c->grid_w)));
    topk = k >= double(1 << 30) ? (1 << 30) : int(k);  // beyond 2^30: every admissible block
  }
  if (topk < 1) return noalloc_fail(LCSA_ERR_INVALID_ARG, "sparse_ratio gives a budget of 0 blocks");
  out->topk = topk;
  out->radius = c->local_range == LCSA_UNBOUNDED ? -1 : (c->local_range - 1) / 2;
  const int groups = g.nKB / g.bpf;
  int wmax = 0;
  int64_t per_head = 0;
  for (int qb = 0; qb < g.nQB; ++qb) {
    const int rem = qb % g.bpf, hb = rem / g.nWb, wb = rem % g.nWb;
    int nh = g.nHb, nw = g.nWb;
    if (out->radius >= 0) {
      const int r = out->radius;
      nh = (hb + r < g.nHb - 1 ? hb + r : g.nHb - 1) - (hb - r > 0 ? hb - r : 0) + 1;
      nw = (wb + r < g.nWb - 1 ? wb + r : g.nWb - 1) - (wb - r > 0 ? wb - r : 0) + 1;
    }
    const int a = groups * nh * nw;
    wmax = a > wmax ? a : wmax;
    per_head += topk < a ? topk : a;
  }
  if (wmax > lcsa::kMaxCandidates) return noalloc_fail(LCSA_ERR_UNSUPPORTED, "window holds too many blocks");
  out->max_window = wmax;
  out->rows = int64_t(g.B) * g.Hn * g.nQB;
  out->nnz = per_head * g.B * g.Hn;
  return LCSA_OK;
}

}  // namespace

extern "C" lcsa_status_t lcsa_forward_noalloc(const lcsa_config_t* cfg, const void* q, const void* k, const void* v,
                                              const float* gamma_q, const float* gamma_k, void* out, void* stream) {
  if (!cfg) return noalloc_fail(LCSA_ERR_INVALID_ARG, "config is null");
  if (cfg->host_io) return noalloc_fail(LCSA_ERR_INVALID_ARG, "host_io needs staging buffers; use a plan");
  if (cfg->heads_total != 0 && cfg->heads_total != cfg->heads)
    return noalloc_fail(LCSA_ERR_UNSUPPORTED, "head-sharded layers need a plan (lcsa_forward_sharded)");
  NoallocGeom ng;
  lcsa_status_t st = noalloc_resolve(cfg, &ng);
  if (st != LCSA_OK) return st;
  if (!q || !k || !v || !gamma_q || !gamma_k || !out) return noalloc_fail(LCSA_ERR_INVALID_ARG, "null tensor pointer");
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out) |
                        reinterpret_cast<uintptr_t>(gamma_q) | reinterpret_cast<uintptr_t>(gamma_k);
  if (mis & 15u) return noalloc_fail(LCSA_ERR_ALIGNMENT, "tensor pointers must be 16-byte aligned");
  const lcsa::Grid& g = ng.g;
  const int radius = ng.radius;
  const int D = cfg->head_dim;

  // carve the static workspace
  const lcsa::RopeSplit rs = lcsa::rope_split(D);
  const size_t rope_n = size_t(g.Tkv) * rs.pairs_t + size_t(g.gh) * rs.pairs_h + size_t(g.gw) * rs.pairs_w;
  const size_t off_err = 0;
  const size_t off_cnt = off_err + 256;  // K1 split counters, cleared together with the error word
  const size_t off_sp = off_cnt + round256(size_t(lcsa::kCounters) * 4);
  const size_t off_rope = off_sp + round256(size_t(lcsa::kMaxK1Ctas) * 2 * g.C * 4);
  const size_t off_rp = off_rope + round256(rope_n * sizeof(float2));
  const size_t off_ci = off_rp + round256((size_t(ng.rows) + 1) * 4);
  const size_t off_pq = off_ci + round256(size_t(ng.nnz) * 4);
  const size_t off_pk = off_pq + round256(size_t(g.B) * g.Hn * g.nQB * D * 4);
  const size_t off_qh = off_pk + round256(size_t(g.B) * g.Hn * g.nKB * D * 4);
  const size_t off_kh = off_qh + round256(size_t(g.B) * g.Lq * g.C * 2);
  // 64-token blocks: query-block pairs as 128-row tiles (union lists and counts)
  const int64_t npairs = g.nb == 64 ? lcsa::pair_count(g) : 0;
  const int pair_cap = 2 * ng.max_window < g.nKB ? 2 * ng.max_window : g.nKB;
  const size_t off_pc = off_kh + round256(size_t(g.B) * g.Lkv * g.C * 2);
  const size_t off_pl = off_pc + round256(size_t(npairs) * size_t(pair_cap) * 4);
  const size_t need = off_pl + round256(size_t(npairs) * 4);
  if (need > size_t(LCSA_NOALLOC_WORKSPACE_BYTES))
    return noalloc_fail(LCSA_ERR_UNSUPPORTED,
                        "problem needs more workspace than the static array holds (LCSA_NOALLOC_WORKSPACE_BYTES); "
                        "create a plan instead");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(LCSA_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(LCSA_ERR_UNSUPPORTED, "device index out of range");
  unsigned char* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_ws_mutex);
    if (!g_ws_addr[dev]) {
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_noalloc_ws);
      if (e != cudaSuccess || !ptr) return noalloc_fail(LCSA_ERR_CUDA, "cudaGetSymbolAddress of the static workspace");
      g_ws_addr[dev] = ptr;
    }
    ws = static_cast<unsigned char*>(g_ws_addr[dev]);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned* err = reinterpret_cast<unsigned*>(ws + off_err);
  unsigned* split_cnt = reinterpret_cast<unsigned*>(ws + off_cnt);
  float* split_part = reinterpret_cast<float*>(ws + off_sp);
  float2* rope = reinterpret_cast<float2*>(ws + off_rope);
  int* row_ptr = reinterpret_cast<int*>(ws + off_rp);
  int* col_idx = reinterpret_cast<int*>(ws + off_ci);
  float* pooled_q = reinterpret_cast<float*>(ws + off_pq);
  float* pooled_k = reinterpret_cast<float*>(ws + off_pk);
  __nv_bfloat16* qhat = reinterpret_cast<__nv_bfloat16*>(ws + off_qh);
  __nv_bfloat16* khat = reinterpret_cast<__nv_bfloat16*>(ws + off_kh);
  int* pair_col = npairs ? reinterpret_cast<int*>(ws + off_pc) : nullptr;
  int* pair_len = npairs ? reinterpret_cast<int*>(ws + off_pl) : nullptr;

  if ((e = cudaMemsetAsync(err, 0, off_sp - off_err, s)) != cudaSuccess)
    return noalloc_fail(LCSA_ERR_CUDA, "clear error word and counters");
  {
    LCSA_RANGE("lcsa rope table");
    if ((e = lcsa::launch_rope_table(rope, g.Tkv, g.gh, g.gw, cfg->kv_frame_offset, D, s)) != cudaSuccess)
      return noalloc_fail(LCSA_ERR_CUDA, "rope table launch");
  }
  noalloc_row_ptr_kernel<<<1, 32, 0, s>>>(row_ptr, g, radius, ng.topk);
  if ((e = cudaGetLastError()) != cudaSuccess) return noalloc_fail(LCSA_ERR_CUDA, "row offsets launch");

  lcsa::K1Params k1{};  // every field zero (null) unless set below
  k1.g = g;
  k1.q = static_cast<const __nv_bfloat16*>(q);
  k1.k = static_cast<const __nv_bfloat16*>(k);
  k1.gamma_q = gamma_q;
  k1.gamma_k = gamma_k;
  k1.qhat = qhat;
  k1.khat = khat;
  k1.pooled_q = pooled_q;
  k1.pooled_k = pooled_k;
  k1.rope = rope;
  k1.rope_h_off = g.Tkv * rs.pairs_t;
  k1.rope_w_off = k1.rope_h_off + g.gh * rs.pairs_h;
  k1.norm_scope = cfg->norm_scope;
  k1.eps = cfg->rms_eps;
  k1.err = err;
  k1.split_part = split_part;
  k1.split_cnt = split_cnt;
  k1.ss_ext = nullptr;
  k1.norm_inv_c = 1.0f / float(g.C);
  lcsa::k1_all_blocks(k1);
  if ((e = cudaDeviceGetAttribute(&k1.num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return noalloc_fail(LCSA_ERR_CUDA, "device attributes");
  {
    LCSA_RANGE("lcsa K1 prologue");
    if ((e = lcsa::launch_prologue(k1, s)) != cudaSuccess) return noalloc_fail(LCSA_ERR_CUDA, "prologue launch");
  }

  int sort_n = 32;
  while (sort_n < ng.max_window) sort_n <<= 1;
  lcsa::K2Params k2{};  // every field zero (null) unless set below
  k2.g = g;
  k2.pooled_q = pooled_q;
  k2.pooled_k = pooled_k;
  k2.row_ptr = row_ptr;
  k2.col_idx = col_idx;
  k2.radius = radius;
  k2.topk = ng.topk;
  k2.sort_n = sort_n;
  k2.clear_cnt = split_cnt;
  k2.n_clear = lcsa::kCounters;
  k2.ring_fb = g.Tkv / g.bt;
  k2.slot0_fb = 0;
  k2.thresh = nullptr;  // no threshold reuse without a plan
  k2.reuse = 0;
  k2.col_pad = nullptr;
  k2.row_len = nullptr;
  k2.pad_cap = 0;
  {
    LCSA_RANGE("lcsa K2 select");
    if ((e = lcsa::launch_select(k2, s)) != cudaSuccess) return noalloc_fail(LCSA_ERR_CUDA, "select launch");
  }
  if (npairs) {
    LCSA_RANGE("lcsa pair union");
    lcsa::PairParams pp{};
    pp.g = g;
    pp.npairs = int(npairs);
    pp.row_ptr = row_ptr;
    pp.col_idx = col_idx;
    pp.nkb = g.nKB;
    pp.pair_col = pair_col;
    pp.pair_len = pair_len;
    pp.pair_cap = pair_cap;
    if ((e = lcsa::launch_pair_union(pp, s)) != cudaSuccess) return noalloc_fail(LCSA_ERR_CUDA, "pair union launch");
  }

  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : float(1.0 / std::sqrt(double(D)));
  lcsa::K3Params k3{};  // every field zero (null) unless set below
  k3.g = g;
  k3.qhat = qhat;
  k3.khat = khat;
  k3.v = static_cast<const __nv_bfloat16*>(v);
  k3.out = static_cast<__nv_bfloat16*>(out);
  k3.row_ptr = row_ptr;
  k3.col_idx = col_idx;
  k3.scale_log2 = scale * 1.4426950408889634f;
  k3.err = err;
  k3.ring_fb = g.Tkv / g.bt;
  k3.slot0_fb = 0;
  k3.row_len = nullptr;
  k3.pad_cap = 0;
  k3.pair_col = pair_col;
  k3.pair_len = pair_len;
  k3.npairs = int(npairs);
  k3.pair_cap = pair_cap;
  k3.work_counter = split_cnt + lcsa::kMaxK1Ctas;
  {
    LCSA_RANGE("lcsa K3 attention");
    CUtensorMap tm_q, tm_k, tm_v;  // encoded on the host stack: no allocation
    const int num_sms = k1.num_sms;
    if ((e = lcsa::make_block_map(&tm_q, qhat, int64_t(g.B) * g.Hn * g.nQB * g.nb, g.nb)) != cudaSuccess ||
        (e = lcsa::make_block_map(&tm_k, khat, int64_t(g.B) * g.Hn * g.nKB * g.nb, g.nb)) != cudaSuccess ||
        (e = lcsa::make_raster_map(&tm_v, v, g)) != cudaSuccess)
      return noalloc_fail(LCSA_ERR_CUDA, "tensor maps");
    if ((e = lcsa::launch_attention_tc(k3, tm_q, tm_k, tm_v, num_sms, s)) != cudaSuccess)
      return noalloc_fail(LCSA_ERR_CUDA, "attention launch");
  }
  return LCSA_OK;
}
