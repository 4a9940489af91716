// Host side of liblcsa: configuration checks, plan (workspace) management and
// the three-kernel forward call. Every entry point returns a status code; no
// path aborts, throws across the ABI or substitutes another implementation.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <array>
#include <vector>

#include "lcsa.h"
#include "lcsa_internal.h"
#include "nvtx_range.h"

namespace {

thread_local std::string g_last_error;

lcsa_status_t fail(lcsa_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

lcsa_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(LCSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

struct Resolved {
  lcsa_geometry_t geo;
  lcsa::Grid grid;
  int radius;          // -1: unbounded
  int sort_n;
  std::vector<int32_t> row_ptr;
  float scale;
  int heads_total;     // heads of the whole (possibly head-sharded) layer
};

// Checks and sizes come from lcsa::resolve_config (lcsa_config.cu), which the
// allocation-free entry point shares; the plan path adds the CSR row offsets
// (they depend on the geometry only) and the workspace size.
lcsa_status_t resolve(const lcsa_config_t* c, Resolved* r, bool want_rows) {
  lcsa::ConfigCore core;
  char why[256];
  const lcsa_status_t st = lcsa::resolve_config(c, &core, why, sizeof(why));
  if (st != LCSA_OK) return fail(st, "%s", why);
  const lcsa::Grid& g = core.grid;
  r->grid = g;
  r->radius = core.radius;
  r->sort_n = core.sort_n;
  r->scale = core.scale;
  r->heads_total = core.heads_total;
  const int64_t rows = core.rows, nnz = core.nnz;
  const int nb = g.nb, wmin = core.min_window, wmax = core.max_window, topk = core.topk;
  if (want_rows) {
    r->row_ptr.assign(size_t(rows) + 1, 0);
    int64_t acc = 0;
    for (int64_t row = 0; row < rows; ++row) {
      r->row_ptr[size_t(row)] = int32_t(acc);
      acc += lcsa::kept_blocks(core, int(row % g.nQB));
    }
    r->row_ptr[size_t(rows)] = int32_t(acc);
  }

  lcsa_geometry_t& o = r->geo;
  std::memset(&o, 0, sizeof(o));
  o.q_tokens = g.Lq;
  o.kv_tokens = g.Lkv;
  o.channels = g.C;
  o.block_tokens = nb;
  o.blocks_per_frame = g.bpf;
  o.q_blocks = g.nQB;
  o.kv_blocks = g.nKB;
  o.rows = rows;
  o.nnz = nnz;
  o.topk = topk;
  o.window_radius = r->radius;
  o.min_window = wmin;
  o.max_window = wmax;
  o.selected_flops = double(nnz) * 4.0 * double(nb) * double(nb) * double(c->head_dim);
  const double act = 2.0 * double(g.C);  // bytes of one bf16 token vector
  o.prologue_bytes = 2.0 * act * double(g.B) * double(g.Lq + g.Lkv);
  // q^ read once, out written once, each (b, h, kept-anywhere) K/V block once
  o.attention_min_bytes = act * double(g.B) * double(2 * g.Lq + 2 * g.Lkv);
  const lcsa::RopeSplit rs = lcsa::rope_split(c->head_dim);
  const size_t rope_n = size_t(g.Tkv) * rs.pairs_t + size_t(g.gh) * rs.pairs_h + size_t(g.gw) * rs.pairs_w;
  size_t ws = 0;
  ws += size_t(g.B) * g.Lq * g.C * 2 + size_t(g.B) * g.Lkv * g.C * 2;            // q^, k^
  ws += size_t(g.B) * g.Hn * (g.nQB + g.nKB) * size_t(c->head_dim) * 4;         // pooled
  ws += (size_t(rows) + 1) * 4 + size_t(nnz) * 4;                                // CSR
  ws += size_t(rows) * (8 + size_t(wmax) * 4);                                    // threshold reuse
  if (nb == 64) {                                                                 // query-block pairs
    const size_t cap = size_t(2 * wmax < g.nKB ? 2 * wmax : g.nKB);
    ws += size_t(lcsa::pair_count(g)) * (cap + 3) * 4;                          // lists, counts, rows
  }
  ws += rope_n * sizeof(float2) + 256;
  ws += size_t(lcsa::kMaxK1Ctas) * 2 * size_t(g.C) * 4 + size_t(lcsa::kCounters) * 4;  // K1 split blocks, counters
  if (nb == 64) {  // merge state of cut pairs, for up to kMaxK1Ctas SMs (the plan sizes it for the device's)
    const size_t cut = size_t(lcsa::cut_items(int(lcsa::pair_count(g)), lcsa::kMaxK1Ctas));
    ws += cut * 8 * 4 + cut * lcsa::kCutParts * 8 * 4 + lcsa::part_buf_floats(int(cut), c->head_dim) * 4;
  }
  if (c->host_io)
    ws += size_t(g.B) * (2 * g.Lq + 2 * g.Lkv) * g.C * 2 + size_t(2) * g.C * 4;
  o.workspace_bytes = ws;
  return LCSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// pair_cap: the union of two query blocks' lists, each at most the largest
// window (a threshold-reuse call can keep a whole window)
int pair_capacity(const Resolved& r) {
  const int two = 2 * r.geo.max_window;
  return two < r.grid.nKB ? two : r.grid.nKB;
}

}  // namespace

struct lcsa_plan {
  lcsa_config_t cfg;
  Resolved res;
  int device = 0;
  __nv_bfloat16* qhat = nullptr;
  __nv_bfloat16* khat = nullptr;
  float* pooled_q = nullptr;
  float* pooled_k = nullptr;
  bool streaming = false;          // made by lcsa_plan_create_stream
  __nv_bfloat16* v_ring = nullptr; // stream plans: raw v of the window, [B][Tkv slots][H'][W'][C]
  int64_t pushed_fb = 0;           // stream plans: frame-blocks pushed so far
  float* split_part = nullptr;     // K1: partial pooled sums of blocks cut between CTAs
  unsigned* split_cnt = nullptr;   // K1: arrivals per cut (K2 zeroes them after use)
  int32_t* row_ptr = nullptr;
  int32_t* col_idx = nullptr;
  // threshold reuse: recorded k-th best scores (order bits) and the padded
  // CSR of reuse calls (max_window entries per row, a count per row)
  unsigned* thresh = nullptr;
  int32_t* row_len = nullptr;
  int32_t* col_pad = nullptr;
  // 64-token blocks: pairs of query blocks as one 128-row tile (union lists)
  int32_t* pair_col = nullptr;
  int32_t* pair_len = nullptr;
  int2* pair_rows = nullptr;
  int npairs = 0, pair_cap = 0;
  // 64-token pairs: merge state of the last pairs, cut into parts
  unsigned* merge_cnt = nullptr;
  unsigned* merge_ready = nullptr;
  float* part_buf = nullptr;
  int cut = 0;
  bool reuse_mode = false;   // lcsa_plan_set_threshold_reuse
  bool have_thresh = false;  // a selecting call has recorded thresholds
  bool last_reuse = false;   // the last call kept blocks by threshold
  float2* rope = nullptr;
  int rope_h_off = 0, rope_w_off = 0;
  unsigned* err = nullptr;
  // host-IO staging
  void* st_q = nullptr;
  void* st_k = nullptr;
  void* st_v = nullptr;
  void* st_out = nullptr;
  float* st_gq = nullptr;
  float* st_gk = nullptr;
  // tcgen05 attention: tensor maps of the plan-owned q^ / k^; SM count (persistent grids)
  CUtensorMap tm_q, tm_k;
  int num_sms = 0;
  // host-IO plans: a copy stream and the events that order it against the
  // call's stream (q/k uploaded, V (or its first half of the heads)
  // uploaded, V's second half uploaded, first attention half done, first
  // half of the output downloaded)
  cudaStream_t io_stream = nullptr;
  cudaEvent_t ev_qk = nullptr, ev_v = nullptr, ev_v2 = nullptr, ev_k3a = nullptr, ev_outa = nullptr;
  unsigned fault_launch = 0;                       // LCSA_FAULT launch:K (kFault* bits)
  bool fault_copy = false;                         // LCSA_FAULT copy
  std::vector<std::array<cudaEvent_t, 4>> evsets;  // timing ring
  int64_t timed = 0;                                // forwards recorded
};

namespace {

void release(lcsa_plan* p) {
  void* ptrs[] = {p->v_ring, p->qhat,  p->khat,    p->pooled_q, p->pooled_k, p->split_part, p->split_cnt,
                  p->row_ptr, p->col_idx, p->rope,     p->err,      p->st_q,       p->st_k,
                  p->st_v,  p->st_out,  p->st_gq,    p->st_gk,    p->thresh,     p->row_len, p->col_pad,
                  p->pair_col, p->pair_len,  p->pair_rows, p->merge_cnt, p->merge_ready, p->part_buf};
  for (void* q : ptrs)
    if (q) cudaFree(q);
  for (auto& set : p->evsets)
    for (auto e : set)
      if (e) cudaEventDestroy(e);
  p->evsets.clear();
  for (cudaEvent_t e : {p->ev_qk, p->ev_v, p->ev_v2, p->ev_k3a, p->ev_outa})
    if (e) cudaEventDestroy(e);
  if (p->io_stream) cudaStreamDestroy(p->io_stream);
}

// Host-side fault injection for tests of the error paths (no GPU fault is
// involved): LCSA_FAULT, read when a plan is created, holds one of
//   alloc:N   the N-th device allocation of that plan's creation fails (OOM)
//   launch:K  every call of the plan reports a failed launch of kernel K
//             (K1, K2, PAIR, K3 or ROPE) instead of launching it
//   copy      lcsa_forward_host reports a failed host-to-device copy
// A value that is none of these refuses the plan (LCSA_ERR_INVALID_ARG), so a
// misspelt injection is never silently ignored.
constexpr unsigned kFaultK1 = 1, kFaultK2 = 2, kFaultPair = 4, kFaultK3 = 8, kFaultRope = 16;
struct Faults {
  int alloc_at = 0;
  unsigned launch = 0;
  bool copy = false;
};
thread_local int t_alloc_countdown = 0;  // > 0 while a plan with alloc:N is being created

lcsa_status_t parse_faults(Faults* f) {
  *f = Faults{};
  const char* v = std::getenv("LCSA_FAULT");
  if (!v || !*v) return LCSA_OK;
  const std::string s(v);
  if (s == "copy") {
    f->copy = true;
    return LCSA_OK;
  }
  if (s.rfind("alloc:", 0) == 0) {
    char* end = nullptr;
    const long n = std::strtol(s.c_str() + 6, &end, 10);
    if (end && *end == 0 && n >= 1 && n <= 1000) {
      f->alloc_at = int(n);
      return LCSA_OK;
    }
  }
  const struct {
    const char* name;
    unsigned bit;
  } kernels[] = {{"launch:K1", kFaultK1}, {"launch:K2", kFaultK2}, {"launch:PAIR", kFaultPair},
                 {"launch:K3", kFaultK3}, {"launch:ROPE", kFaultRope}};
  for (const auto& k : kernels)
    if (s == k.name) {
      f->launch = k.bit;
      return LCSA_OK;
    }
  return fail(LCSA_ERR_INVALID_ARG, "LCSA_FAULT=%s not understood (alloc:N, launch:K1|K2|PAIR|K3|ROPE, copy)", v);
}

lcsa_status_t injected_launch_failure(const lcsa_plan* p, unsigned bit, const char* what) {
  return (p->fault_launch & bit) ? fail(LCSA_ERR_CUDA, "%s launch: injected failure (LCSA_FAULT)", what) : LCSA_OK;
}

template <class T>
lcsa_status_t dev_alloc(T** ptr, size_t bytes, const char* what) {
  if (t_alloc_countdown > 0 && --t_alloc_countdown == 0) {
    *ptr = nullptr;
    return fail(LCSA_ERR_OOM, "cudaMalloc(%s, %zu bytes): injected failure (LCSA_FAULT)", what, bytes);
  }
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(ptr), bytes < 16 ? 16 : bytes);
  if (e != cudaSuccess) {
    *ptr = nullptr;
    cudaGetLastError();
    return fail(e == cudaErrorMemoryAllocation ? LCSA_ERR_OOM : LCSA_ERR_CUDA, "cudaMalloc(%s, %zu bytes): %s", what,
                bytes, cudaGetErrorString(e));
  }
  return LCSA_OK;
}

lcsa_status_t alloc_pairs(lcsa_plan* p) {
  const int64_t np = lcsa::pair_count(p->res.grid);
  if (np > (int64_t(1) << 30)) return fail(LCSA_ERR_UNSUPPORTED, "%lld query-block pairs", (long long)np);
  p->npairs = int(np);
  p->pair_cap = pair_capacity(p->res);
  lcsa_status_t st = dev_alloc(&p->pair_col, size_t(np) * size_t(p->pair_cap) * 4, "pair lists");
  if (st == LCSA_OK) st = dev_alloc(&p->pair_len, size_t(np) * 4, "pair counts");
  if (st == LCSA_OK) st = dev_alloc(&p->pair_rows, size_t(np) * sizeof(int2), "pair rows");
  // the last pairs are cut into parts: the attention's merge state
  p->cut = lcsa::cut_items(p->npairs, p->num_sms);
  const size_t cut = size_t(p->cut);
  if (st == LCSA_OK) st = dev_alloc(&p->merge_cnt, cut * 8 * 4, "cut pairs' counters");
  if (st == LCSA_OK) st = dev_alloc(&p->merge_ready, cut * lcsa::kCutParts * 8 * 4, "cut pairs' ready flags");
  if (st == LCSA_OK) st = dev_alloc(&p->part_buf, lcsa::part_buf_floats(p->cut, p->res.grid.D) * 4, "cut pairs' partials");
  return st;
}

// Read the plan's device error word (the stream is already synchronised),
// clear it if set, and map it to a status.
lcsa_status_t take_device_error(lcsa_plan* p) {
  unsigned word[4] = {0, 0, 0, 0};
  cudaError_t e = cudaMemcpy(word, p->err, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  if (word[0] == lcsa::kDevErrNone) return LCSA_OK;
  if ((e = cudaMemset(p->err, 0, 256)) != cudaSuccess) return cuda_fail(e, "clear error word");
  if (word[0] == lcsa::kDevErrTimeout)
    return fail(LCSA_ERR_DEVICE_TIMEOUT, "kernel gave up a bounded wait (site %u, block %u)", word[1], word[2]);
  return fail(LCSA_ERR_DEVICE_BOUNDS, "kernel index check failed (site %u, value %u)", word[1], word[2]);
}

}  // namespace

extern "C" {

void lcsa_config_default(lcsa_config_t* c) {
  if (!c) return;
  std::memset(c, 0, sizeof(*c));
  c->batch = 1;
  c->heads = 12;
  c->head_dim = 128;
  c->q_frames = 2;
  c->kv_frames = 6;
  c->grid_h = 48;
  c->grid_w = 80;
  c->block_t = 1;
  c->block_h = 8;
  c->block_w = 16;
  c->local_range = 11;
  c->topk = 0;
  c->sparse_ratio = 2.0f;
  c->kv_frame_offset = 0;
  c->norm_scope = LCSA_NORM_TOKEN;
  c->rms_eps = 1e-6f;
  c->softmax_scale = 0.f;
  c->host_io = 0;
}

lcsa_status_t lcsa_config_resolve(const lcsa_config_t* cfg, lcsa_geometry_t* out) {
  if (!out) return fail(LCSA_ERR_INVALID_ARG, "geometry output is null");
  Resolved r;
  lcsa_status_t st = resolve(cfg, &r, false);
  if (st == LCSA_OK) *out = r.geo;
  return st;
}

}  // extern "C"

namespace {

// Validate, allocate and set up a plan (the allocations count down
// t_alloc_countdown, set by the callers from LCSA_FAULT).
lcsa_status_t create_plan(const lcsa_config_t* cfg, int cuda_device, const Faults& faults, lcsa_plan_t* out) {
  lcsa_plan* p = new (std::nothrow) lcsa_plan();
  if (!p) return fail(LCSA_ERR_OOM, "host allocation of the plan");
  lcsa_status_t st = resolve(cfg, &p->res, true);
  if (st != LCSA_OK) {
    delete p;
    return st;
  }
  p->cfg = *cfg;
  p->device = cuda_device;
  p->fault_launch = faults.launch;
  p->fault_copy = faults.copy;
  cudaError_t e = cudaSetDevice(cuda_device);
  if (e != cudaSuccess) {
    delete p;
    cudaGetLastError();
    return cuda_fail(e, "cudaSetDevice");
  }
  const lcsa::Grid& g = p->res.grid;
  const lcsa::RopeSplit rs = lcsa::rope_split(cfg->head_dim);
  const size_t rope_n = size_t(g.Tkv) * rs.pairs_t + size_t(g.gh) * rs.pairs_h + size_t(g.gw) * rs.pairs_w;
  p->rope_h_off = g.Tkv * rs.pairs_t;
  p->rope_w_off = p->rope_h_off + g.gh * rs.pairs_h;
  const size_t rows = size_t(p->res.geo.rows), nnz = size_t(p->res.geo.nnz);
  const size_t D = size_t(cfg->head_dim);
  if ((e = cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, cuda_device)) != cudaSuccess) {
    delete p;
    return cuda_fail(e, "device attributes");
  }
  if ((st = dev_alloc(&p->qhat, size_t(g.B) * g.Lq * g.C * 2, "q^")) ||
      (st = dev_alloc(&p->khat, size_t(g.B) * g.Lkv * g.C * 2, "k^")) ||
      (st = dev_alloc(&p->pooled_q, size_t(g.B) * g.Hn * g.nQB * D * 4, "pooled q")) ||
      (st = dev_alloc(&p->pooled_k, size_t(g.B) * g.Hn * g.nKB * D * 4, "pooled k")) ||
      (st = dev_alloc(&p->row_ptr, (rows + 1) * 4, "row_ptr")) ||
      (st = dev_alloc(&p->col_idx, nnz * 4, "col_idx")) ||
      (st = dev_alloc(&p->thresh, rows * 4, "thresholds")) ||
      (st = dev_alloc(&p->row_len, rows * 4, "row counts")) ||
      (st = dev_alloc(&p->col_pad, rows * size_t(p->res.geo.max_window) * 4, "padded col_idx")) ||
      (g.nb == 64 && (st = alloc_pairs(p)) != LCSA_OK) ||
      (st = dev_alloc(&p->rope, rope_n * sizeof(float2), "rope table")) ||
      (st = dev_alloc(&p->err, 256, "error word")) ||
      (st = dev_alloc(&p->split_part, size_t(lcsa::kMaxK1Ctas) * 2 * g.C * 4, "K1 split sums")) ||
      (st = dev_alloc(&p->split_cnt, size_t(lcsa::kCounters) * 4, "K1 split and K3 work counters"))) {
    release(p);
    delete p;
    return st;
  }
  if (cfg->host_io) {
    if ((st = dev_alloc(&p->st_q, size_t(g.B) * g.Lq * g.C * 2, "staging q")) ||
        (st = dev_alloc(&p->st_k, size_t(g.B) * g.Lkv * g.C * 2, "staging k")) ||
        (st = dev_alloc(&p->st_v, size_t(g.B) * g.Lkv * g.C * 2, "staging v")) ||
        (st = dev_alloc(&p->st_out, size_t(g.B) * g.Lq * g.C * 2, "staging out")) ||
        (st = dev_alloc(&p->st_gq, size_t(g.C) * 4, "staging gamma q")) ||
        (st = dev_alloc(&p->st_gk, size_t(g.C) * 4, "staging gamma k"))) {
      release(p);
      delete p;
      return st;
    }
    if ((e = cudaStreamCreateWithFlags(&p->io_stream, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&p->ev_qk, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&p->ev_v, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&p->ev_v2, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&p->ev_k3a, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&p->ev_outa, cudaEventDisableTiming)) != cudaSuccess) {
      release(p);
      delete p;
      return cuda_fail(e, "host-IO stream and events");
    }
  }
  if ((e = cudaMemcpy(p->row_ptr, p->res.row_ptr.data(), (rows + 1) * 4, cudaMemcpyHostToDevice)) != cudaSuccess ||
      (e = cudaMemset(p->err, 0, 256)) != cudaSuccess ||
      (e = cudaMemset(p->split_cnt, 0, size_t(lcsa::kCounters) * 4)) != cudaSuccess ||
      (e = lcsa::launch_rope_table(p->rope, g.Tkv, g.gh, g.gw, cfg->kv_frame_offset, cfg->head_dim, 0)) !=
          cudaSuccess ||
      (e = cudaDeviceSynchronize()) != cudaSuccess) {
    release(p);
    delete p;
    return cuda_fail(e, "plan set-up");
  }
  {
    if ((e = lcsa::make_block_map(&p->tm_q, p->qhat, int64_t(g.B) * g.Hn * g.nQB * g.nb, g.nb, g.D)) != cudaSuccess ||
        (e = lcsa::make_block_map(&p->tm_k, p->khat, int64_t(g.B) * g.Hn * g.nKB * g.nb, g.nb, g.D)) != cudaSuccess) {
      release(p);
      delete p;
      return cuda_fail(e, "tensor maps");
    }
  }
  *out = p;
  return LCSA_OK;
}

}  // namespace

extern "C" {

lcsa_status_t lcsa_plan_create(const lcsa_config_t* cfg, int cuda_device, lcsa_plan_t* out) {
  if (!out) return fail(LCSA_ERR_INVALID_ARG, "plan output is null");
  *out = nullptr;
  Faults faults;
  lcsa_status_t st = parse_faults(&faults);
  if (st != LCSA_OK) return st;
  t_alloc_countdown = faults.alloc_at;
  st = create_plan(cfg, cuda_device, faults, out);
  t_alloc_countdown = 0;
  return st;
}

void lcsa_plan_destroy(lcsa_plan_t p) {
  if (!p) return;
  cudaSetDevice(p->device);
  cudaDeviceSynchronize();
  release(p);
  delete p;
}

namespace {

// Which frames one launch sequence covers. The stateless call: the whole
// window from the caller's tensors. A stream step: `fb` new frame-blocks of
// k (and v, copied into the plan's ring first), the chunk's queries when q is
// given, and the ring slot of window frame-block 0.
struct StepBlocks {
  bool with_q = true;   // run K1 on q, then K2 and K3
  int k_in_fb = 0;      // frame-blocks of the k input
  int k_first_fb = 0;   // window frame-block of the k input's first one
  int slot0_fb = 0;     // ring slot of window frame-block 0
  const void* v_attn = nullptr;  // raster v seen by K3 (caller's tensor or the ring)
  const float* ss_ext = nullptr; // head-sharded token-scope norm: reduced per-token sums of squares
  cudaEvent_t k3_wait = nullptr; // an event K3 waits for (the host-IO call's V upload)
  int k3_split = 0;              // > 0: K3 as two launches, work items [0, k3_split) and the rest,
  cudaEvent_t k3_first_done = nullptr;  // recorded between them
  cudaEvent_t k3_wait_b = nullptr;      // an event the second of them also waits for (V's second half)
};

lcsa_status_t run_step(lcsa_plan_t p, const void* q, const void* k, const float* gamma_q, const float* gamma_k,
                       void* out, cudaStream_t s, const StepBlocks& sb) {
  const lcsa::Grid& g = p->res.grid;
  cudaError_t e;
  lcsa::K1Params k1{};  // every field zero (null) unless set below
  k1.g = g;
  k1.q = static_cast<const __nv_bfloat16*>(q);
  k1.k = static_cast<const __nv_bfloat16*>(k);
  k1.gamma_q = gamma_q;
  k1.gamma_k = gamma_k;
  k1.qhat = p->qhat;
  k1.khat = p->khat;
  k1.pooled_q = p->pooled_q;
  k1.pooled_k = p->pooled_k;
  k1.rope = p->rope;
  k1.rope_h_off = p->rope_h_off;
  k1.rope_w_off = p->rope_w_off;
  k1.norm_scope = p->cfg.norm_scope;
  k1.eps = p->cfg.rms_eps;
  k1.err = p->err;
  k1.num_sms = p->num_sms;
  k1.split_part = p->split_part;
  k1.split_cnt = p->split_cnt;
  k1.n_qblk = sb.with_q ? g.B * g.nQB : 0;
  k1.k_in_fb = sb.k_in_fb;
  k1.k_first_fb = sb.k_first_fb;
  k1.ring_fb = g.Tkv / g.bt;
  k1.slot0_fb = sb.slot0_fb;
  k1.Lk_in = int64_t(sb.k_in_fb) * g.bt * g.gh * g.gw;
  k1.ss_ext = sb.ss_ext;
  k1.norm_inv_c = 1.0f / float(int64_t(p->res.heads_total) * g.D);

  lcsa::K2Params k2{};  // every field zero (null) unless set below
  k2.g = g;
  k2.pooled_q = p->pooled_q;
  k2.pooled_k = p->pooled_k;
  k2.row_ptr = p->row_ptr;
  k2.col_idx = p->col_idx;
  k2.radius = p->res.radius;
  k2.topk = p->res.geo.topk;
  k2.sort_n = p->res.sort_n;
  k2.clear_cnt = p->split_cnt;
  k2.n_clear = lcsa::kCounters;
  k2.ring_fb = g.Tkv / g.bt;
  k2.slot0_fb = sb.slot0_fb;
  const bool reuse = p->reuse_mode && p->have_thresh;
  k2.thresh = p->thresh;
  k2.reuse = reuse ? 1 : 0;
  k2.col_pad = p->col_pad;
  k2.row_len = p->row_len;
  k2.pad_cap = p->res.geo.max_window;

  lcsa::K3Params k3{};  // every field zero (null) unless set below
  k3.g = g;
  k3.qhat = p->qhat;
  k3.khat = p->khat;
  k3.v = static_cast<const __nv_bfloat16*>(sb.v_attn);
  k3.out = static_cast<__nv_bfloat16*>(out);
  k3.row_ptr = p->row_ptr;
  k3.col_idx = reuse ? p->col_pad : p->col_idx;
  k3.row_len = reuse ? p->row_len : nullptr;
  k3.pad_cap = p->res.geo.max_window;
  k3.npairs = p->npairs;
  k3.pair_col = p->pair_col;
  k3.pair_len = p->pair_len;
  k3.pair_rows = p->pair_rows;
  k3.pair_cap = p->pair_cap;
  k3.work_counter = p->split_cnt + lcsa::kMaxK1Ctas;
  k3.cut_items = p->cut;
  k3.merge_cnt = p->merge_cnt;
  k3.merge_ready = p->merge_ready;
  k3.part_buf = p->part_buf;
  k3.scale_log2 = p->res.scale * 1.4426950408889634f;
  k3.err = p->err;
  k3.ring_fb = g.Tkv / g.bt;
  k3.slot0_fb = sb.slot0_fb;

  cudaEvent_t* ev = nullptr;
  if (sb.with_q && !p->evsets.empty()) ev = p->evsets[size_t(p->timed % int64_t(p->evsets.size()))].data();
  if (ev && (e = cudaEventRecord(ev[0], s)) != cudaSuccess) return cuda_fail(e, "event");
  {
    LCSA_RANGE("lcsa K1 prologue");
    if (lcsa_status_t st = injected_launch_failure(p, kFaultK1, "prologue")) return st;
    if ((e = lcsa::launch_prologue(k1, s)) != cudaSuccess) return cuda_fail(e, "prologue launch");
  }
  if (!sb.with_q) {
    // no K2 after this K1: clear its merge counters here
    if ((e = cudaMemsetAsync(p->split_cnt, 0, size_t(lcsa::kCounters) * 4, s)) != cudaSuccess)
      return cuda_fail(e, "clear merge counters");
    return LCSA_OK;
  }
  if (ev && (e = cudaEventRecord(ev[1], s)) != cudaSuccess) return cuda_fail(e, "event");
  {
    LCSA_RANGE("lcsa K2 select");
    if (lcsa_status_t st = injected_launch_failure(p, kFaultK2, "select")) return st;
    if ((e = lcsa::launch_select(k2, s)) != cudaSuccess) return cuda_fail(e, "select launch");
  }
  if (p->pair_col) {
    LCSA_RANGE("lcsa pair union");
    lcsa::PairParams pp{};
    pp.g = g;
    pp.npairs = p->npairs;
    pp.row_ptr = p->row_ptr;
    pp.col_idx = reuse ? p->col_pad : p->col_idx;
    pp.row_len = reuse ? p->row_len : nullptr;
    pp.pad_cap = p->res.geo.max_window;
    pp.nkb = g.nKB;
    pp.pair_col = p->pair_col;
    pp.pair_len = p->pair_len;
    pp.pair_rows = p->pair_rows;
    pp.pair_cap = p->pair_cap;
    pp.merge_cnt = p->merge_cnt;
    pp.merge_ready = p->merge_ready;
    pp.cut = p->cut;
    if (lcsa_status_t st = injected_launch_failure(p, kFaultPair, "pair union")) return st;
    if ((e = lcsa::launch_pair_union(pp, s)) != cudaSuccess) return cuda_fail(e, "pair union launch");
  }
  p->have_thresh = true;
  p->last_reuse = reuse;
  if (ev && (e = cudaEventRecord(ev[2], s)) != cudaSuccess) return cuda_fail(e, "event");
  {
    LCSA_RANGE("lcsa K3 attention");
    CUtensorMap tm_v;
    if ((e = lcsa::make_raster_map(&tm_v, sb.v_attn, g)) != cudaSuccess) return cuda_fail(e, "V tensor map");
    if (lcsa_status_t st = injected_launch_failure(p, kFaultK3, "attention")) return st;
    if (sb.k3_wait && (e = cudaStreamWaitEvent(s, sb.k3_wait, 0)) != cudaSuccess) return cuda_fail(e, "wait for V");
    if (sb.k3_split > 0) {
      // two launches over the two halves of the work items, each with its own
      // zeroed work counter; the event between them lets the caller start on
      // the first half's output
      k3.item_lo = 0;
      k3.item_hi = sb.k3_split;
      if ((e = lcsa::launch_attention_tc(k3, p->tm_q, p->tm_k, tm_v, p->num_sms, s)) != cudaSuccess)
        return cuda_fail(e, "attention launch");
      if ((e = cudaEventRecord(sb.k3_first_done, s)) != cudaSuccess) return cuda_fail(e, "event");
      k3.item_lo = sb.k3_split;
      k3.item_hi = 0;  // to the end
      k3.work_counter += 1;
      if (sb.k3_wait_b && (e = cudaStreamWaitEvent(s, sb.k3_wait_b, 0)) != cudaSuccess)
        return cuda_fail(e, "wait for V");
    }
    if ((e = lcsa::launch_attention_tc(k3, p->tm_q, p->tm_k, tm_v, p->num_sms, s)) != cudaSuccess)
      return cuda_fail(e, "attention launch");
  }
  if (ev) {
    if ((e = cudaEventRecord(ev[3], s)) != cudaSuccess) return cuda_fail(e, "event");
    ++p->timed;
  }
  return LCSA_OK;
}

}  // namespace

namespace {

bool sharded_token_norm(lcsa_plan_t p) {
  return p->res.heads_total > p->res.grid.Hn && p->cfg.norm_scope == LCSA_NORM_TOKEN;
}

lcsa_status_t forward_common(lcsa_plan_t p, const void* q, const void* k, const void* v, const float* gamma_q,
                             const float* gamma_k, const float* ssq, void* out, void* stream) {
  if (!q || !k || !v || !gamma_q || !gamma_k || !out) return fail(LCSA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(gamma_q) ||
      !aligned16(gamma_k))
    return fail(LCSA_ERR_ALIGNMENT, "tensor pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSetDevice(p->device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  const lcsa::Grid& g = p->res.grid;
  StepBlocks sb;
  sb.k_in_fb = g.Tkv / g.bt;
  sb.v_attn = v;
  sb.ss_ext = ssq;
  return run_step(p, q, k, gamma_q, gamma_k, out, s, sb);
}

}  // namespace

lcsa_status_t lcsa_forward(lcsa_plan_t p, const void* q, const void* k, const void* v, const float* gamma_q,
                           const float* gamma_k, void* out, void* stream) {
  if (!p) return fail(LCSA_ERR_INVALID_ARG, "plan is null");
  if (p->streaming) return fail(LCSA_ERR_INVALID_ARG, "a stream plan takes lcsa_forward_stream");
  if (sharded_token_norm(p))
    return fail(LCSA_ERR_INVALID_ARG, "a head-sharded plan with token-scope norm takes lcsa_forward_sharded");
  return forward_common(p, q, k, v, gamma_q, gamma_k, nullptr, out, stream);
}

lcsa_status_t lcsa_sumsq(lcsa_plan_t p, const void* q, const void* k, float* ssq, void* stream) {
  if (!p) return fail(LCSA_ERR_INVALID_ARG, "plan is null");
  if (p->streaming) return fail(LCSA_ERR_INVALID_ARG, "stream plans are not head-sharded");
  if (!q || !k || !ssq) return fail(LCSA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(ssq))
    return fail(LCSA_ERR_ALIGNMENT, "tensor pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSetDevice(p->device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  const lcsa::Grid& g = p->res.grid;
  const int64_t nq = int64_t(g.B) * g.Lq, nk = int64_t(g.B) * g.Lkv;
  LCSA_RANGE("lcsa sumsq");
  if ((e = lcsa::launch_sumsq(static_cast<const __nv_bfloat16*>(q), nq, static_cast<const __nv_bfloat16*>(k), nk,
                              g.C, ssq, s)) != cudaSuccess)
    return cuda_fail(e, "sum of squares launch");
  return LCSA_OK;
}

lcsa_status_t lcsa_forward_sharded(lcsa_plan_t p, const void* q, const void* k, const void* v, const float* gamma_q,
                                   const float* gamma_k, const float* ssq, void* out, void* stream) {
  if (!p) return fail(LCSA_ERR_INVALID_ARG, "plan is null");
  if (p->streaming) return fail(LCSA_ERR_INVALID_ARG, "stream plans are not head-sharded");
  if (!ssq) return fail(LCSA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(ssq)) return fail(LCSA_ERR_ALIGNMENT, "tensor pointers must be 16-byte aligned");
  if (p->cfg.norm_scope != LCSA_NORM_TOKEN)
    return fail(LCSA_ERR_INVALID_ARG, "head-scope norm needs no exchange: use lcsa_forward");
  return forward_common(p, q, k, v, gamma_q, gamma_k, ssq, out, stream);
}

lcsa_status_t lcsa_plan_create_stream(const lcsa_config_t* cfg, int cuda_device, lcsa_plan_t* out) {
  if (cfg && cfg->host_io) return fail(LCSA_ERR_INVALID_ARG, "stream plans take device tensors (host_io = 0)");
  if (cfg && cfg->heads_total != 0 && cfg->heads_total != cfg->heads)
    return fail(LCSA_ERR_UNSUPPORTED, "stream plans are not head-sharded");
  if (!out) return fail(LCSA_ERR_INVALID_ARG, "plan output is null");
  *out = nullptr;
  Faults faults;
  lcsa_status_t st = parse_faults(&faults);
  if (st != LCSA_OK) return st;
  t_alloc_countdown = faults.alloc_at;
  st = create_plan(cfg, cuda_device, faults, out);
  if (st != LCSA_OK) {
    t_alloc_countdown = 0;
    return st;
  }
  lcsa_plan* p = *out;
  const lcsa::Grid& g = p->res.grid;
  st = dev_alloc(&p->v_ring, size_t(g.B) * g.Lkv * g.C * 2, "v ring");
  t_alloc_countdown = 0;
  if (st != LCSA_OK) {
    lcsa_plan_destroy(p);
    *out = nullptr;
    return st;
  }
  p->streaming = true;
  p->pushed_fb = 0;
  return LCSA_OK;
}

namespace {

// One stream step: `frames` new frames of k and v (and the chunk's q when
// given) enter the window; the ring slot of absolute frame-block F is
// F % (Tkv / bt). Copies v into the ring, rebuilds the frame RoPE table for
// the window's new absolute position, then runs the kernels.
lcsa_status_t stream_step(lcsa_plan_t p, const void* q, const void* k, const void* v, const float* gamma_q,
                          const float* gamma_k, int frames, void* out, cudaStream_t s) {
  const lcsa::Grid& g = p->res.grid;
  const int ring = g.Tkv / g.bt;
  if (frames <= 0 || frames % g.bt || frames > g.Tkv)
    return fail(LCSA_ERR_SHAPE, "%d frames (a multiple of block_t, at most kv_frames = %d)", frames, g.Tkv);
  cudaError_t e = cudaSetDevice(p->device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  const int fb = frames / g.bt;
  const int64_t after = p->pushed_fb + fb;
  if (q && after < ring)
    return fail(LCSA_ERR_INVALID_ARG, "the KV window is not full yet (%lld of %d frame-blocks): push frames first",
                (long long)after, ring);
  const size_t frame_bytes = size_t(g.gh) * g.gw * g.C * 2;
  for (int b = 0; b < g.B; ++b)
    for (int f = 0; f < frames; ++f) {
      const int64_t abs_fb = p->pushed_fb + f / g.bt;
      const int slot = int(abs_fb % ring);
      char* dst = reinterpret_cast<char*>(p->v_ring) + (size_t(b) * g.Tkv + size_t(slot) * g.bt + f % g.bt) * frame_bytes;
      const char* src = static_cast<const char*>(v) + (size_t(b) * frames + f) * frame_bytes;
      if ((e = cudaMemcpyAsync(dst, src, frame_bytes, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
        return cuda_fail(e, "v ring copy");
    }
  const int64_t w0_fb = after - ring;  // window frame-block 0, counted from the first push (may be < 0)
  const int t0 = p->cfg.kv_frame_offset + int(w0_fb) * g.bt;
  {
    LCSA_RANGE("lcsa rope table");
    if (lcsa_status_t st = injected_launch_failure(p, kFaultRope, "rope table")) return st;
    if ((e = lcsa::launch_rope_table(p->rope, g.Tkv, g.gh, g.gw, t0, p->cfg.head_dim, s)) != cudaSuccess)
      return cuda_fail(e, "rope table launch");
  }
  StepBlocks sb;
  sb.with_q = q != nullptr;
  sb.k_in_fb = fb;
  sb.k_first_fb = ring - fb;
  sb.slot0_fb = int(((w0_fb % ring) + ring) % ring);
  sb.v_attn = p->v_ring;
  lcsa_status_t st = run_step(p, q ? q : k, k, q ? gamma_q : gamma_k, gamma_k, out, s, sb);
  if (st == LCSA_OK) p->pushed_fb = after;
  return st;
}

}  // namespace

lcsa_status_t lcsa_stream_push(lcsa_plan_t p, const void* k, const void* v, const float* gamma_k, int frames,
                               void* stream) {
  if (!p) return fail(LCSA_ERR_INVALID_ARG, "plan is null");
  if (!p->streaming) return fail(LCSA_ERR_INVALID_ARG, "not a stream plan (lcsa_plan_create_stream)");
  if (!k || !v || !gamma_k) return fail(LCSA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(k) || !aligned16(v) || !aligned16(gamma_k))
    return fail(LCSA_ERR_ALIGNMENT, "tensor pointers must be 16-byte aligned");
  return stream_step(p, nullptr, k, v, nullptr, gamma_k, frames, nullptr, static_cast<cudaStream_t>(stream));
}

lcsa_status_t lcsa_forward_stream(lcsa_plan_t p, const void* q, const void* k, const void* v, const float* gamma_q,
                                  const float* gamma_k, void* out, void* stream) {
  if (!p) return fail(LCSA_ERR_INVALID_ARG, "plan is null");
  if (!p->streaming) return fail(LCSA_ERR_INVALID_ARG, "not a stream plan (lcsa_plan_create_stream)");
  if (!q || !k || !v || !gamma_q || !gamma_k || !out) return fail(LCSA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(gamma_q) ||
      !aligned16(gamma_k))
    return fail(LCSA_ERR_ALIGNMENT, "tensor pointers must be 16-byte aligned");
  return stream_step(p, q, k, v, gamma_q, gamma_k, p->res.grid.Tq, out, static_cast<cudaStream_t>(stream));
}

lcsa_status_t lcsa_forward_host(lcsa_plan_t p, const void* q, const void* k, const void* v, const float* gamma_q,
                                const float* gamma_k, void* out, void* stream) {
  if (!p) return fail(LCSA_ERR_INVALID_ARG, "plan is null");
  if (!p->cfg.host_io) return fail(LCSA_ERR_INVALID_ARG, "plan was created without host_io");
  if (sharded_token_norm(p))
    return fail(LCSA_ERR_INVALID_ARG, "a head-sharded plan with token-scope norm takes lcsa_forward_sharded");
  if (!q || !k || !v || !gamma_q || !gamma_k || !out) return fail(LCSA_ERR_INVALID_ARG, "null host pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSetDevice(p->device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  const lcsa::Grid& g = p->res.grid;
  const size_t qb = size_t(g.B) * g.Lq * g.C * 2, kb = size_t(g.B) * g.Lkv * g.C * 2, gb = size_t(g.C) * 4;
  if (p->fault_copy) return fail(LCSA_ERR_CUDA, "host-to-device copy: injected failure (LCSA_FAULT)");
  // With one batch element and at least two heads K3 runs as two launches
  // over the first and the second half of the heads (rows, or query-block
  // pairs, are numbered head-major): each reads only its heads' channels of
  // v, so v goes up in those two halves (strided copies, a token's channels
  // being head-major) and each launch waits only for its own; the first
  // half's output channels go back on the copy stream while the second half
  // computes.
  const int heads_a = g.B == 1 && g.Hn >= 2 ? g.Hn / 2 : 0;
  const size_t pitch = size_t(g.C) * 2, head_bytes = size_t(g.D) * 2;
  // The copies share one link, so they go in the order the kernels need
  // them: gains, q and k on the call's stream (K1 and K2 start as soon as
  // they are in), then v on the plan's copy stream while K1 and K2 run.
  if ((e = cudaMemcpyAsync(p->st_gq, gamma_q, gb, cudaMemcpyHostToDevice, s)) != cudaSuccess ||
      (e = cudaMemcpyAsync(p->st_gk, gamma_k, gb, cudaMemcpyHostToDevice, s)) != cudaSuccess ||
      (e = cudaMemcpyAsync(p->st_q, q, qb, cudaMemcpyHostToDevice, s)) != cudaSuccess ||
      (e = cudaMemcpyAsync(p->st_k, k, kb, cudaMemcpyHostToDevice, s)) != cudaSuccess ||
      (e = cudaEventRecord(p->ev_qk, s)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(p->io_stream, p->ev_qk, 0)) != cudaSuccess)
    return cuda_fail(e, "host-to-device copy");
  if (heads_a > 0) {
    char* dv = static_cast<char*>(p->st_v);
    const char* hv = static_cast<const char*>(v);
    if ((e = cudaMemcpy2DAsync(dv, pitch, hv, pitch, heads_a * head_bytes, size_t(g.Lkv), cudaMemcpyHostToDevice,
                               p->io_stream)) != cudaSuccess ||
        (e = cudaEventRecord(p->ev_v, p->io_stream)) != cudaSuccess ||
        (e = cudaMemcpy2DAsync(dv + heads_a * head_bytes, pitch, hv + heads_a * head_bytes, pitch,
                               (g.Hn - heads_a) * head_bytes, size_t(g.Lkv), cudaMemcpyHostToDevice,
                               p->io_stream)) != cudaSuccess ||
        (e = cudaEventRecord(p->ev_v2, p->io_stream)) != cudaSuccess)
      return cuda_fail(e, "host-to-device copy");
  } else if ((e = cudaMemcpyAsync(p->st_v, v, kb, cudaMemcpyHostToDevice, p->io_stream)) != cudaSuccess ||
             (e = cudaEventRecord(p->ev_v, p->io_stream)) != cudaSuccess) {
    return cuda_fail(e, "host-to-device copy");
  }
  StepBlocks sb;
  sb.k_in_fb = g.Tkv / g.bt;
  sb.v_attn = p->st_v;
  sb.k3_wait = p->ev_v;
  if (heads_a > 0) {
    const int64_t per_head = p->pair_col ? lcsa::pair_count(g) / g.Hn : int64_t(g.nQB);
    sb.k3_split = int(heads_a * per_head);
    sb.k3_first_done = p->ev_k3a;
    sb.k3_wait_b = p->ev_v2;
  }
  lcsa_status_t st = run_step(p, p->st_q, p->st_k, p->st_gq, p->st_gk, p->st_out, s, sb);
  if (st != LCSA_OK) return st;
  if (heads_a > 0) {
    if ((e = cudaStreamWaitEvent(p->io_stream, p->ev_k3a, 0)) != cudaSuccess ||
        (e = cudaMemcpy2DAsync(out, pitch, p->st_out, pitch, heads_a * head_bytes, size_t(g.Lq),
                               cudaMemcpyDeviceToHost, p->io_stream)) != cudaSuccess ||
        (e = cudaEventRecord(p->ev_outa, p->io_stream)) != cudaSuccess ||
        (e = cudaMemcpy2DAsync(static_cast<char*>(out) + heads_a * head_bytes, pitch,
                               static_cast<const char*>(static_cast<const void*>(p->st_out)) + heads_a * head_bytes,
                               pitch, (g.Hn - heads_a) * head_bytes, size_t(g.Lq), cudaMemcpyDeviceToHost, s)) !=
            cudaSuccess ||
        (e = cudaStreamWaitEvent(s, p->ev_outa, 0)) != cudaSuccess)
      return cuda_fail(e, "device-to-host copy");
  } else if ((e = cudaMemcpyAsync(out, p->st_out, qb, cudaMemcpyDeviceToHost, s)) != cudaSuccess) {
    return cuda_fail(e, "device-to-host copy");
  }
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "stream synchronize");
  return take_device_error(p);
}

lcsa_status_t lcsa_plan_geometry(lcsa_plan_t p, lcsa_geometry_t* out) {
  if (!p || !out) return fail(LCSA_ERR_INVALID_ARG, "null argument");
  *out = p->res.geo;
  return LCSA_OK;
}

lcsa_status_t lcsa_plan_topk(lcsa_plan_t p, int* k_out) {
  if (!p || !k_out) return fail(LCSA_ERR_INVALID_ARG, "null argument");
  *k_out = p->res.geo.topk;
  return LCSA_OK;
}

lcsa_status_t lcsa_plan_set_threshold_reuse(lcsa_plan_t p, int on) {
  if (!p) return fail(LCSA_ERR_INVALID_ARG, "plan is null");
  if (on != 0 && on != 1) return fail(LCSA_ERR_INVALID_ARG, "on = %d (0 or 1)", on);
  p->reuse_mode = on != 0;
  return LCSA_OK;
}

lcsa_status_t lcsa_selection_nnz(lcsa_plan_t p, int64_t* nnz) {
  if (!p || !nnz) return fail(LCSA_ERR_INVALID_ARG, "null argument");
  if (!p->last_reuse) {
    *nnz = p->res.geo.nnz;
    return LCSA_OK;
  }
  const size_t rows = size_t(p->res.geo.rows);
  std::vector<int32_t> len(rows);
  cudaError_t e = cudaSetDevice(p->device);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(len.data(), p->row_len, rows * 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "copy row counts");
  int64_t n = 0;
  for (int32_t v : len) n += v;
  *nnz = n;
  return LCSA_OK;
}

lcsa_status_t lcsa_get_selection(lcsa_plan_t p, int32_t* row_ptr, size_t row_ptr_cap, int32_t* col_idx,
                                 size_t col_idx_cap) {
  if (!p || !row_ptr || !col_idx) return fail(LCSA_ERR_INVALID_ARG, "null argument");
  if (p->last_reuse) {
    // the padded CSR of a reuse call, compacted on the host
    const size_t rows = size_t(p->res.geo.rows), cap = size_t(p->res.geo.max_window);
    std::vector<int32_t> len(rows), pad(rows * cap);
    cudaError_t e = cudaSetDevice(p->device);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(len.data(), p->row_len, rows * 4, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(pad.data(), p->col_pad, rows * cap * 4, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "copy selection");
    size_t n = 0;
    for (size_t r = 0; r < rows; ++r) n += size_t(len[r]);
    if (row_ptr_cap < rows + 1 || col_idx_cap < n)
      return fail(LCSA_ERR_INVALID_ARG, "capacity %zu/%zu < %zu/%zu", row_ptr_cap, col_idx_cap, rows + 1, n);
    row_ptr[0] = 0;
    for (size_t r = 0; r < rows; ++r) {
      if (len[r] < 0 || size_t(len[r]) > cap) return fail(LCSA_ERR_DEVICE_BOUNDS, "row %zu count %d", r, len[r]);
      std::memcpy(col_idx + row_ptr[r], pad.data() + r * cap, size_t(len[r]) * 4);
      row_ptr[r + 1] = row_ptr[r] + len[r];
    }
    return LCSA_OK;
  }
  const size_t rows = size_t(p->res.geo.rows), nnz = size_t(p->res.geo.nnz);
  if (row_ptr_cap < rows + 1 || col_idx_cap < nnz)
    return fail(LCSA_ERR_INVALID_ARG, "capacity %zu/%zu < %zu/%zu", row_ptr_cap, col_idx_cap, rows + 1, nnz);
  cudaError_t e = cudaSetDevice(p->device);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(row_ptr, p->row_ptr, (rows + 1) * 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(col_idx, p->col_idx, nnz * 4, cudaMemcpyDeviceToHost);
  return e == cudaSuccess ? LCSA_OK : cuda_fail(e, "copy selection");
}

lcsa_status_t lcsa_get_intermediates(lcsa_plan_t p, void* qhat, void* khat, float* pooled_q, float* pooled_k) {
  if (!p) return fail(LCSA_ERR_INVALID_ARG, "plan is null");
  const lcsa::Grid& g = p->res.grid;
  cudaError_t e = cudaSetDevice(p->device);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess && qhat) e = cudaMemcpy(qhat, p->qhat, size_t(g.B) * g.Lq * g.C * 2, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && khat) e = cudaMemcpy(khat, p->khat, size_t(g.B) * g.Lkv * g.C * 2, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && pooled_q)
    e = cudaMemcpy(pooled_q, p->pooled_q, size_t(g.B) * g.Hn * g.nQB * g.D * 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && pooled_k)
    e = cudaMemcpy(pooled_k, p->pooled_k, size_t(g.B) * g.Hn * g.nKB * g.D * 4, cudaMemcpyDeviceToHost);
  return e == cudaSuccess ? LCSA_OK : cuda_fail(e, "copy intermediates");
}

lcsa_status_t lcsa_check_device_error(lcsa_plan_t p, void* stream) {
  if (!p) return fail(LCSA_ERR_INVALID_ARG, "plan is null");
  cudaError_t e = cudaSetDevice(p->device);
  if (e == cudaSuccess) e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream");
  return take_device_error(p);
}

lcsa_status_t lcsa_plan_set_timing(lcsa_plan_t p, int capacity) {
  if (!p) return fail(LCSA_ERR_INVALID_ARG, "plan is null");
  if (capacity < 0 || capacity > (1 << 16)) return fail(LCSA_ERR_INVALID_ARG, "timing capacity %d", capacity);
  cudaError_t e = cudaSetDevice(p->device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  for (auto& set : p->evsets)
    for (auto ev : set) cudaEventDestroy(ev);
  p->evsets.clear();
  p->timed = 0;
  for (int i = 0; i < capacity; ++i) {
    std::array<cudaEvent_t, 4> set{};
    for (auto& ev : set) {
      if ((e = cudaEventCreate(&ev)) != cudaSuccess) {
        p->evsets.push_back(set);
        return cuda_fail(e, "cudaEventCreate");
      }
    }
    p->evsets.push_back(set);
  }
  return LCSA_OK;
}

lcsa_status_t lcsa_get_kernel_times(lcsa_plan_t p, float ms[3], int* count) {
  if (!p || !ms) return fail(LCSA_ERR_INVALID_ARG, "null argument");
  if (p->evsets.empty() || p->timed == 0) return fail(LCSA_ERR_INVALID_ARG, "no timed forward recorded");
  const int64_t cap = int64_t(p->evsets.size());
  const int64_t n = p->timed < cap ? p->timed : cap;
  cudaError_t e = cudaEventSynchronize(p->evsets[size_t((p->timed - 1) % cap)][3]);
  double acc[3] = {0, 0, 0};
  for (int64_t i = 0; i < n && e == cudaSuccess; ++i) {
    const auto& set = p->evsets[size_t((p->timed - 1 - i) % cap)];
    for (int k = 0; k < 3 && e == cudaSuccess; ++k) {
      float t = 0.f;
      e = cudaEventElapsedTime(&t, set[k], set[k + 1]);
      acc[k] += t;
    }
  }
  if (e != cudaSuccess) return cuda_fail(e, "event timing");
  for (int k = 0; k < 3; ++k) ms[k] = float(acc[k] / double(n));
  if (count) *count = int(n);
  return LCSA_OK;
}

lcsa_status_t lcsa_selftest_exp2(const float* x, float* y, int n, void* stream) {
  if (!x || !y || n < 0) return fail(LCSA_ERR_INVALID_ARG, "null pointer or negative count");
  if (n == 0) return LCSA_OK;
  cudaError_t e = lcsa::launch_exp2_selftest(x, y, n, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LCSA_OK : cuda_fail(e, "exp2 self-test launch");
}

const char* lcsa_status_string(lcsa_status_t s) {
  switch (s) {
    case LCSA_OK: return "LCSA_OK";
    case LCSA_ERR_INVALID_ARG: return "LCSA_ERR_INVALID_ARG";
    case LCSA_ERR_SHAPE: return "LCSA_ERR_SHAPE";
    case LCSA_ERR_ALIGNMENT: return "LCSA_ERR_ALIGNMENT";
    case LCSA_ERR_UNSUPPORTED: return "LCSA_ERR_UNSUPPORTED";
    case LCSA_ERR_OOM: return "LCSA_ERR_OOM";
    case LCSA_ERR_CUDA: return "LCSA_ERR_CUDA";
    case LCSA_ERR_DEVICE_TIMEOUT: return "LCSA_ERR_DEVICE_TIMEOUT";
    case LCSA_ERR_DEVICE_BOUNDS: return "LCSA_ERR_DEVICE_BOUNDS";
  }
  return "LCSA_ERR_UNKNOWN";
}

const char* lcsa_last_error_message(void) { return g_last_error.c_str(); }

int lcsa_abi_version(void) { return LCSA_ABI_VERSION; }

}  // extern "C"
