// Configuration checks and derived sizes, shared by the plan path
// (lcsa_config_resolve, lcsa_plan_create) and the allocation-free path
// (lcsa_forward_noalloc): one set of rules, so the two cannot drift apart.
// Host code only; it touches no device and no heap (a failure reason is
// formatted only into a buffer the caller passes).
//
// The budget rule follows the "FlashVSR Inference" skill, Non-Negotiable
// Streaming Contract: topk_ratio = sparse_ratio * 768 * 1280 / (H * W) with the
// pixel size H = 16 grid_h, W = 16 grid_w, read as a fraction of the blocks of
// one latent frame and floored. The window is an odd, centred diameter in
// blocks ("FlashVSR - Real-Time Diffusion-Based Video Super-Resolution", How it
// works: attention limited to local patches), clipped at the frame edge.
#include <cmath>
#include <cstdarg>
#include <cstdio>

#include "lcsa.h"
#include "lcsa_internal.h"

namespace lcsa {
namespace {

lcsa_status_t refuse(char* msg, size_t cap, lcsa_status_t st, const char* fmt, ...) {
  if (msg && cap) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(msg, cap, fmt, ap);
    va_end(ap);
  }
  return st;
}

// Blocks of one axis inside the window of a block at `center` (all n when
// the window is unbounded).
int span(int center, int rad, int n) {
  if (rad < 0) return n;
  const int lo = center - rad < 0 ? 0 : center - rad;
  const int hi = center + rad > n - 1 ? n - 1 : center + rad;
  return hi - lo + 1;
}

}  // namespace

int budget_from_ratio(double sparse_ratio, int gh, int gw, int64_t blocks_per_frame) {
  const double pixels = (16.0 * gh) * (16.0 * gw);
  const double k = std::floor(sparse_ratio * 983040.0 * double(blocks_per_frame) / pixels);
  return k >= double(1 << 30) ? (1 << 30) : int(k);
}

int window_blocks(const ConfigCore& r, int qb) {
  const Grid& g = r.grid;
  const int rem = qb % g.bpf;
  return (g.nKB / g.bpf) * span(rem / g.nWb, r.radius, g.nHb) * span(rem % g.nWb, r.radius, g.nWb);
}

int kept_blocks(const ConfigCore& r, int qb) {
  const int a = window_blocks(r, qb);
  return r.topk < a ? r.topk : a;
}

lcsa_status_t resolve_config(const lcsa_config_t* c, ConfigCore* r, char* msg, size_t cap) {
  if (!c) return refuse(msg, cap, LCSA_ERR_INVALID_ARG, "config is null");
  if (c->batch < 1 || c->heads < 1 || c->head_dim < 1 || c->q_frames < 1 || c->kv_frames < 1 || c->grid_h < 1 ||
      c->grid_w < 1 || c->block_t < 1 || c->block_h < 1 || c->block_w < 1)
    return refuse(msg, cap, LCSA_ERR_INVALID_ARG, "sizes must be >= 1");
  if (c->local_range < 0 || (c->local_range != LCSA_UNBOUNDED && c->local_range % 2 == 0))
    return refuse(msg, cap, LCSA_ERR_INVALID_ARG,
                  "local_range %d must be odd (a centred window diameter) or 0 (unbounded)", c->local_range);
  if (c->topk < 0) return refuse(msg, cap, LCSA_ERR_INVALID_ARG, "topk %d < 0", c->topk);
  if (c->topk == 0 && !(c->sparse_ratio > 0.f && std::isfinite(c->sparse_ratio)))
    return refuse(msg, cap, LCSA_ERR_INVALID_ARG, "topk = 0 needs a finite sparse_ratio > 0");
  if (c->norm_scope != LCSA_NORM_TOKEN && c->norm_scope != LCSA_NORM_HEAD)
    return refuse(msg, cap, LCSA_ERR_INVALID_ARG, "norm_scope %d", c->norm_scope);
  if (!(c->rms_eps > 0.f) || !std::isfinite(c->rms_eps))
    return refuse(msg, cap, LCSA_ERR_INVALID_ARG, "rms_eps must be finite and > 0");
  if (!(c->softmax_scale >= 0.f) || !std::isfinite(c->softmax_scale))
    return refuse(msg, cap, LCSA_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  if (c->kv_frame_offset < 0) return refuse(msg, cap, LCSA_ERR_INVALID_ARG, "kv_frame_offset < 0");
  if (c->kv_frames < c->q_frames)
    return refuse(msg, cap, LCSA_ERR_SHAPE,
                  "kv_frames %d < q_frames %d (queries are the last frames of the KV window)", c->kv_frames,
                  c->q_frames);
  if (c->grid_h % c->block_h || c->grid_w % c->block_w || c->q_frames % c->block_t || c->kv_frames % c->block_t)
    return refuse(msg, cap, LCSA_ERR_SHAPE, "token grid %dx%dx%d (q %d) not divisible by block %dx%dx%d",
                  c->kv_frames, c->grid_h, c->grid_w, c->q_frames, c->block_t, c->block_h, c->block_w);
  if (c->head_dim != 64 && c->head_dim != 128)
    return refuse(msg, cap, LCSA_ERR_UNSUPPORTED, "head_dim %d (64 or 128)", c->head_dim);
  if (c->heads > kMaxHeads) return refuse(msg, cap, LCSA_ERR_UNSUPPORTED, "heads %d > %d", c->heads, kMaxHeads);
  const int nb = c->block_t * c->block_h * c->block_w;
  if (nb != 64 && nb != 128) return refuse(msg, cap, LCSA_ERR_UNSUPPORTED, "block of %d tokens (64 or 128)", nb);
  if (c->block_t * c->block_h > 8)
    return refuse(msg, cap, LCSA_ERR_UNSUPPORTED, "block_t*block_h = %d > 8 token rows", c->block_t * c->block_h);
  if (c->heads_total != 0 && c->heads_total < c->heads)
    return refuse(msg, cap, LCSA_ERR_INVALID_ARG, "heads_total %d < heads %d", c->heads_total, c->heads);
  // bound the sizes (in floating point, so nothing below can overflow): at
  // most 2^40 elements per tensor, hence at most 2^33 tokens and 2^27 blocks,
  // which every int block count and int64 token index holds
  const double elems_max = double(c->batch) * double(c->kv_frames) * double(c->grid_h) * double(c->grid_w) *
                           double(c->heads) * double(c->head_dim);
  if (elems_max > double(int64_t(1) << 40))
    return refuse(msg, cap, LCSA_ERR_UNSUPPORTED, "tensor of %.4g elements (> 2^40)", elems_max);

  Grid& g = r->grid;
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
  g.D = c->head_dim;
  g.C = c->heads * c->head_dim;
  r->heads_total = c->heads_total == 0 ? c->heads : c->heads_total;

  r->rows = int64_t(g.B) * g.Hn * g.nQB;
  if (r->rows > (int64_t(1) << 30)) return refuse(msg, cap, LCSA_ERR_UNSUPPORTED, "%lld rows", (long long)r->rows);

  int topk = c->topk;
  if (topk == 0) {
    topk = budget_from_ratio(double(c->sparse_ratio), c->grid_h, c->grid_w, g.bpf);
    if (topk < 1)
      return refuse(msg, cap, LCSA_ERR_INVALID_ARG, "sparse_ratio %g gives a budget of %d blocks",
                    double(c->sparse_ratio), topk);
  }
  r->topk = topk;
  r->radius = c->local_range == LCSA_UNBOUNDED ? -1 : (c->local_range - 1) / 2;

  // admissible-set sizes: they depend on the block's place in its frame only,
  // so one frame group's blocks give every query block's
  int wmin = 1 << 30, wmax = 0;
  int64_t per_frame = 0;
  for (int rem = 0; rem < g.bpf; ++rem) {
    const int a = window_blocks(*r, rem);
    wmin = a < wmin ? a : wmin;
    wmax = a > wmax ? a : wmax;
    per_frame += topk < a ? topk : a;
  }
  if (wmax > kMaxCandidates)
    return refuse(msg, cap, LCSA_ERR_UNSUPPORTED, "window holds %d blocks (> %d)", wmax, kMaxCandidates);
  r->min_window = wmin;
  r->max_window = wmax;
  int sort_n = 32;
  while (sort_n < wmax) sort_n <<= 1;
  r->sort_n = sort_n;
  const int64_t nnz = per_frame * (g.nQB / g.bpf) * g.B * g.Hn;
  if (nnz > (int64_t(1) << 31) - 1) return refuse(msg, cap, LCSA_ERR_UNSUPPORTED, "%lld kept blocks", (long long)nnz);
  r->nnz = nnz;
  r->scale = c->softmax_scale > 0.f ? c->softmax_scale : float(1.0 / std::sqrt(double(c->head_dim)));
  return LCSA_OK;
}

}  // namespace lcsa
