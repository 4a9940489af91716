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
// This entry point runs the same kernels with every intermediate placed in a
// file-scope static device array of LCSA_NOALLOC_WORKSPACE_BYTES, and the
// configuration goes through the same checks as a plan's (resolve_config).
//
// Set-up: the first call in a CUDA context looks up the array's device address
// there (cudaGetSymbolAddress with that context current) and clears its error
// word. Under CUDA's default lazy module loading that lookup is also what
// loads this file's module, and loading it reserves the array on the device:
// make the first call at start-up, before any stream capture (or load every
// module at start-up with CUDA_MODULE_LOADING=EAGER). Later calls allocate
// nothing. The address is cached per context (by its unique context ID), so a
// context created later on the same device, for instance after
// cudaDeviceReset, looks it up again.
//
// All calls share the one array and it keeps the last call's contents, so
// calls that overlap on the GPU (other streams, other host threads) race;
// serialise them. Each call clears the counters its kernels start from; the
// kernels overwrite every other byte they read. The error word is not
// cleared by a call: a kernel's timeout or bounds record stays until
// lcsa_noalloc_check_device_error reads it.
#include <cmath>
#include <mutex>

#include "lcsa.h"
#include "lcsa_internal.h"
#include "nvtx_range.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_ws[LCSA_NOALLOC_WORKSPACE_BYTES];

// Layout of the array's first bytes: the error word (kept across calls),
// then K1's merge counters and K3's work counter (cleared by every call).
constexpr size_t kOffErr = 0;
constexpr size_t kOffCnt = 256;
constexpr size_t round256(size_t n) { return (n + 255) & ~size_t(255); }
constexpr size_t kOffAfterCnt = kOffCnt + round256(size_t(lcsa::kCounters) * 4);

// Workspace address per CUDA context, keyed by the context's unique ID
// (cuCtxGetId; IDs are never reused within a process).
constexpr int kMaxContexts = 64;
struct WsEntry {
  unsigned long long ctx_id;
  unsigned char* addr;
};
std::mutex g_ws_mutex;
WsEntry g_ws[kMaxContexts] = {};
int g_ws_n = 0;

using CtxGetCurrent = CUresult (*)(CUcontext*);
using CtxGetId = CUresult (*)(CUcontext, unsigned long long*);

// ID of the calling thread's current context (false if there is none).
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrent get_current = nullptr;
  static CtxGetId get_id = nullptr;
  if (!get_current || !get_id) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess)
      return false;
    get_current = reinterpret_cast<CtxGetCurrent>(f1);
    get_id = reinterpret_cast<CtxGetId>(f2);
  }
  CUcontext ctx = nullptr;
  return get_current(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, id) == CUDA_SUCCESS;
}

// The array's address in the current context, looked up (and its error word
// cleared on `s`) the first time. Caller holds g_ws_mutex. Null on failure.
unsigned char* workspace_here(cudaStream_t s, bool set_up) {
  unsigned long long id = 0;
  if (!current_context_id(&id)) return nullptr;
  for (int i = 0; i < g_ws_n; ++i)
    if (g_ws[i].ctx_id == id) return g_ws[i].addr;
  if (!set_up || g_ws_n == kMaxContexts) return nullptr;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_ws) != cudaSuccess || !ptr) return nullptr;
  if (cudaMemsetAsync(static_cast<unsigned char*>(ptr) + kOffErr, 0, kOffCnt - kOffErr, s) != cudaSuccess)
    return nullptr;
  g_ws[g_ws_n++] = WsEntry{id, static_cast<unsigned char*>(ptr)};
  return static_cast<unsigned char*>(ptr);
}

// CSR row offsets from the geometry alone. A query block's kept count
// depends only on its place in its frame, so the block first scans the kept
// counts of one frame's places into pre[0..bpf] (1024 at a time, warp scans
// and a carry), then writes row (bh, qb) = bh * per_head + (qb / bpf) *
// per_frame + pre[qb % bpf].
__global__ void __launch_bounds__(1024) noalloc_row_ptr_kernel(int* row_ptr, int* pre, lcsa::ConfigCore r) {
  __shared__ int warp_incl[32];
  __shared__ int carry;
  const lcsa::Grid& g = r.grid;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < g.bpf; base += 1024) {
    const int place = base + tid;
    int v = 0;
    if (place < g.bpf) {
      const int hb = place / g.nWb, wb = place % g.nWb;
      int nh = g.nHb, nw = g.nWb;
      if (r.radius >= 0) {
        nh = min(hb + r.radius, g.nHb - 1) - max(hb - r.radius, 0) + 1;
        nw = min(wb + r.radius, g.nWb - 1) - max(wb - r.radius, 0) + 1;
      }
      const int a = (g.nKB / g.bpf) * nh * nw;
      v = r.topk < a ? r.topk : a;
    }
    int x = v;  // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_incl[w] = x;
    __syncthreads();
    if (w == 0) {
      int t = warp_incl[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      warp_incl[lane] = t;
    }
    __syncthreads();
    const int excl = carry + (w > 0 ? warp_incl[w - 1] : 0) + x - v;
    if (place < g.bpf) pre[place] = excl;
    __syncthreads();  // every thread has read carry
    if (tid == 1023) carry = excl + v;
    __syncthreads();
  }
  const int per_frame = carry;
  const int64_t per_head = int64_t(per_frame) * (g.nQB / g.bpf);
  const int rows = g.B * g.Hn * g.nQB;
  for (int row = tid; row < rows; row += 1024) {
    const int bh = row / g.nQB, qb = row % g.nQB;
    row_ptr[row] = int(bh * per_head + int64_t(qb / g.bpf) * per_frame + pre[qb % g.bpf]);
  }
  if (tid == 0) row_ptr[rows] = int(int64_t(g.B) * g.Hn * per_head);
}

}  // namespace

extern "C" lcsa_status_t lcsa_forward_noalloc(const lcsa_config_t* cfg, const void* q, const void* k, const void* v,
                                              const float* gamma_q, const float* gamma_k, void* out, void* stream) {
  // Failures are reported by status code only: composing a message string
  // could allocate host memory, which this entry point never does.
  if (!cfg) return LCSA_ERR_INVALID_ARG;
  if (cfg->host_io) return LCSA_ERR_INVALID_ARG;  // host buffers need staging: use a plan
  if (cfg->heads_total != 0 && cfg->heads_total != cfg->heads)
    return LCSA_ERR_UNSUPPORTED;  // head-sharded layers need a plan (lcsa_forward_sharded)
  lcsa::ConfigCore core;
  lcsa_status_t st = lcsa::resolve_config(cfg, &core, nullptr, 0);
  if (st != LCSA_OK) return st;
  if (!q || !k || !v || !gamma_q || !gamma_k || !out) return LCSA_ERR_INVALID_ARG;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out) |
                        reinterpret_cast<uintptr_t>(gamma_q) | reinterpret_cast<uintptr_t>(gamma_k);
  if (mis & 15u) return LCSA_ERR_ALIGNMENT;
  const lcsa::Grid& g = core.grid;
  const int D = cfg->head_dim;

  // carve the static workspace
  const lcsa::RopeSplit rs = lcsa::rope_split(D);
  const size_t rope_n = size_t(g.Tkv) * rs.pairs_t + size_t(g.gh) * rs.pairs_h + size_t(g.gw) * rs.pairs_w;
  const size_t off_sp = kOffAfterCnt;
  const size_t off_rope = off_sp + round256(size_t(lcsa::kMaxK1Ctas) * 2 * g.C * 4);
  const size_t off_pre = off_rope + round256(rope_n * sizeof(float2));
  const size_t off_rp = off_pre + round256((size_t(g.bpf) + 1) * 4);
  const size_t off_ci = off_rp + round256((size_t(core.rows) + 1) * 4);
  const size_t off_pq = off_ci + round256(size_t(core.nnz) * 4);
  const size_t off_pk = off_pq + round256(size_t(g.B) * g.Hn * g.nQB * D * 4);
  const size_t off_qh = off_pk + round256(size_t(g.B) * g.Hn * g.nKB * D * 4);
  const size_t off_kh = off_qh + round256(size_t(g.B) * g.Lq * g.C * 2);
  // 64-token blocks: query-block pairs as 128-row tiles (union lists, counts and rows)
  const int64_t npairs = g.nb == 64 ? lcsa::pair_count(g) : 0;
  const int pair_cap = 2 * core.max_window < g.nKB ? 2 * core.max_window : g.nKB;
  const size_t off_pc = off_kh + round256(size_t(g.B) * g.Lkv * g.C * 2);
  const size_t off_pl = off_pc + round256(size_t(npairs) * size_t(pair_cap) * 4);
  const size_t off_pr = off_pl + round256(size_t(npairs) * 4);
  const size_t off_sg = off_pr + round256(size_t(npairs) * sizeof(int2));
  // the problem's own buffers must fit before any device is asked anything
  if (off_sg > size_t(LCSA_NOALLOC_WORKSPACE_BYTES)) return LCSA_ERR_UNSUPPORTED;  // create a plan instead
  int dev = 0, num_sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return LCSA_ERR_CUDA;
  if ((e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return LCSA_ERR_CUDA;
  // 64-token pairs: the attention's merge state of the last pairs, cut into parts
  const int cut = npairs ? lcsa::cut_items(int(npairs), num_sms) : 0;
  const size_t off_mc = off_sg;
  const size_t off_mr = off_mc + round256(size_t(cut) * 8 * 4);
  const size_t off_pb = off_mr + round256(size_t(cut) * lcsa::kCutParts * 8 * 4);
  const size_t need = off_pb + round256(lcsa::part_buf_floats(cut, D) * 4);
  if (need > size_t(LCSA_NOALLOC_WORKSPACE_BYTES)) return LCSA_ERR_UNSUPPORTED;  // create a plan instead
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_ws_mutex);
    ws = workspace_here(s, true);
  }
  if (!ws) return LCSA_ERR_CUDA;
  unsigned* err = reinterpret_cast<unsigned*>(ws + kOffErr);
  unsigned* split_cnt = reinterpret_cast<unsigned*>(ws + kOffCnt);
  float* split_part = reinterpret_cast<float*>(ws + off_sp);
  float2* rope = reinterpret_cast<float2*>(ws + off_rope);
  int* pre = reinterpret_cast<int*>(ws + off_pre);
  int* row_ptr = reinterpret_cast<int*>(ws + off_rp);
  int* col_idx = reinterpret_cast<int*>(ws + off_ci);
  float* pooled_q = reinterpret_cast<float*>(ws + off_pq);
  float* pooled_k = reinterpret_cast<float*>(ws + off_pk);
  __nv_bfloat16* qhat = reinterpret_cast<__nv_bfloat16*>(ws + off_qh);
  __nv_bfloat16* khat = reinterpret_cast<__nv_bfloat16*>(ws + off_kh);
  int* pair_col = npairs ? reinterpret_cast<int*>(ws + off_pc) : nullptr;
  int* pair_len = npairs ? reinterpret_cast<int*>(ws + off_pl) : nullptr;
  int2* pair_rows = npairs ? reinterpret_cast<int2*>(ws + off_pr) : nullptr;
  unsigned* merge_cnt = reinterpret_cast<unsigned*>(ws + off_mc);
  unsigned* merge_ready = reinterpret_cast<unsigned*>(ws + off_mr);
  float* part_buf = reinterpret_cast<float*>(ws + off_pb);

  // the counters start at zero (an aborted call may have left them set)
  if ((e = cudaMemsetAsync(split_cnt, 0, kOffAfterCnt - kOffCnt, s)) != cudaSuccess) return LCSA_ERR_CUDA;
  {
    LCSA_RANGE("lcsa rope table");
    if ((e = lcsa::launch_rope_table(rope, g.Tkv, g.gh, g.gw, cfg->kv_frame_offset, D, s)) != cudaSuccess)
      return LCSA_ERR_CUDA;
  }
  noalloc_row_ptr_kernel<<<1, 1024, 0, s>>>(row_ptr, pre, core);
  if ((e = cudaGetLastError()) != cudaSuccess) return LCSA_ERR_CUDA;

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
  k1.num_sms = num_sms;
  {
    LCSA_RANGE("lcsa K1 prologue");
    if ((e = lcsa::launch_prologue(k1, s)) != cudaSuccess) return LCSA_ERR_CUDA;
  }

  lcsa::K2Params k2{};  // every field zero (null) unless set below
  k2.g = g;
  k2.pooled_q = pooled_q;
  k2.pooled_k = pooled_k;
  k2.row_ptr = row_ptr;
  k2.col_idx = col_idx;
  k2.radius = core.radius;
  k2.topk = core.topk;
  k2.sort_n = core.sort_n;
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
    if ((e = lcsa::launch_select(k2, s)) != cudaSuccess) return LCSA_ERR_CUDA;
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
    pp.pair_rows = pair_rows;
    pp.pair_cap = pair_cap;
    pp.merge_cnt = merge_cnt;
    pp.merge_ready = merge_ready;
    pp.cut = cut;
    if ((e = lcsa::launch_pair_union(pp, s)) != cudaSuccess) return LCSA_ERR_CUDA;
  }

  lcsa::K3Params k3{};  // every field zero (null) unless set below
  k3.g = g;
  k3.qhat = qhat;
  k3.khat = khat;
  k3.v = static_cast<const __nv_bfloat16*>(v);
  k3.out = static_cast<__nv_bfloat16*>(out);
  k3.row_ptr = row_ptr;
  k3.col_idx = col_idx;
  k3.scale_log2 = core.scale * 1.4426950408889634f;
  k3.err = err;
  k3.ring_fb = g.Tkv / g.bt;
  k3.slot0_fb = 0;
  k3.row_len = nullptr;
  k3.pad_cap = 0;
  k3.pair_col = pair_col;
  k3.pair_len = pair_len;
  k3.pair_rows = pair_rows;
  k3.npairs = int(npairs);
  k3.pair_cap = pair_cap;
  k3.work_counter = split_cnt + lcsa::kMaxK1Ctas;
  k3.cut_items = cut;
  k3.merge_cnt = merge_cnt;
  k3.merge_ready = merge_ready;
  k3.part_buf = part_buf;
  {
    LCSA_RANGE("lcsa K3 attention");
    CUtensorMap tm_q, tm_k, tm_v;  // encoded on the host stack: no allocation
    if ((e = lcsa::make_block_map(&tm_q, qhat, int64_t(g.B) * g.Hn * g.nQB * g.nb, g.nb, g.D)) != cudaSuccess ||
        (e = lcsa::make_block_map(&tm_k, khat, int64_t(g.B) * g.Hn * g.nKB * g.nb, g.nb, g.D)) != cudaSuccess ||
        (e = lcsa::make_raster_map(&tm_v, v, g)) != cudaSuccess)
      return LCSA_ERR_CUDA;
    if ((e = lcsa::launch_attention_tc(k3, tm_q, tm_k, tm_v, num_sms, s)) != cudaSuccess) return LCSA_ERR_CUDA;
  }
  return LCSA_OK;
}

extern "C" lcsa_status_t lcsa_noalloc_check_device_error(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_ws_mutex);
    ws = workspace_here(s, false);
  }
  if (!ws) return LCSA_OK;  // no call has run in this context
  if (cudaStreamSynchronize(s) != cudaSuccess) return LCSA_ERR_CUDA;
  unsigned word[4] = {0, 0, 0, 0};  // host stack: no allocation
  if (cudaMemcpy(word, ws + kOffErr, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return LCSA_ERR_CUDA;
  if (word[0] == lcsa::kDevErrNone) return LCSA_OK;
  if (cudaMemset(ws + kOffErr, 0, sizeof(word)) != cudaSuccess) return LCSA_ERR_CUDA;
  return word[0] == lcsa::kDevErrTimeout ? LCSA_ERR_DEVICE_TIMEOUT : LCSA_ERR_DEVICE_BOUNDS;
}
