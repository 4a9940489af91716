// Internal interface between the host side of liblcsa (plan, validation,
// launches) and the three kernels. Not installed; the public ABI is lcsa.h.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lcsa.h"

namespace lcsa {

constexpr int kMaxHeadDim = 128;     // head sizes the kernels implement: 64 and 128
constexpr int kMaxHeads = 16;
constexpr int kMaxCandidates = 4096; // admissible blocks per query block (K2 sort)
constexpr int kMaxK1Ctas = 256;      // K1 persistent grid cap (sizes its split-block buffers)
// The plan's counter array: K1's kMaxK1Ctas merge counters, then K3's two
// work counters (a call may run K3 as two launches over halves of the work
// items); K2 zeroes all of them (after K1 has used its own, before K3 starts).
constexpr int kCounters = kMaxK1Ctas + 2;

// Device error word codes (first word of the plan's error buffer).
constexpr unsigned kDevErrNone = 0;
constexpr unsigned kDevErrTimeout = 1;
constexpr unsigned kDevErrBounds = 2;

// Factored 3D RoPE split of a head: pairs [0, pairs_t) follow the frame,
// [pairs_t, pairs_t + pairs_h) the token row, the rest the token column.
struct RopeSplit {
  int pairs_t, pairs_h, pairs_w;
  int dims_t, dims_h, dims_w;
};
inline RopeSplit rope_split(int d) {
  RopeSplit s;
  s.dims_h = 2 * (d / 6);
  s.dims_w = 2 * (d / 6);
  s.dims_t = d - s.dims_h - s.dims_w;
  s.pairs_t = s.dims_t / 2;
  s.pairs_h = s.dims_h / 2;
  s.pairs_w = s.dims_w / 2;
  return s;
}

// Geometry shared by all kernels (token grid, blocks, window).
struct Grid {
  int B, Hn;            // batch, heads
  int Tq, Tkv;          // query / KV frames
  int gh, gw;           // token grid per frame
  int bt, bh, bw;       // block shape
  int nb;               // tokens per block
  int nHb, nWb, bpf;    // block rows / columns / blocks per frame group
  int nQB, nKB;         // blocks per (batch, head)
  int64_t Lq, Lkv;      // tokens per batch element
  int D;                // head_dim (64 or 128)
  int C;                // heads * head_dim
};

struct K1Params {
  Grid g;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const float* gamma_q;
  const float* gamma_k;
  __nv_bfloat16* qhat;  // [B][Hn][nQB][nb][d]
  __nv_bfloat16* khat;  // [B][Hn][nKB][nb][d]
  float* pooled_q;      // [B][Hn][nQB][d]
  float* pooled_k;      // [B][Hn][nKB][d]
  const float2* rope;   // cos/sin: [Tkv][pairs_t], [gh][pairs_h], [gw][pairs_w]
  int rope_h_off, rope_w_off;  // float2 offsets of the row and column tables
  int norm_scope;       // 0 token, 1 head
  float eps;
  unsigned* err;        // device error word (bounded waits record a timeout here)
  int num_sms;          // persistent grid size (one CTA per SM, at most kMaxK1Ctas)
  float* split_part;    // [kMaxK1Ctas][2][C] partial pooled sums of blocks cut between CTAs
  unsigned* split_cnt;  // [kMaxK1Ctas] arrivals per cut; zero on entry (K2 clears them)
  // Which blocks this launch processes. A stateless call: all of q and k
  // (n_qblk = B nQB, k_in_fb = ring_fb, k_first_fb = slot0_fb = 0). A stream
  // call: the new frames only, k^ / pooled k written to the ring slots
  // ((slot0_fb + window frame-block) % ring_fb).
  int n_qblk;           // query blocks processed: B * nQB, or 0 (a KV-only push)
  int k_in_fb;          // frame-blocks of the k input (its frames / bt)
  int k_first_fb;       // KV-window frame-block of the k input's first frame-block
  int ring_fb;          // KV window length in frame-blocks (Tkv / bt)
  int slot0_fb;         // ring slot of window frame-block 0
  int64_t Lk_in;        // tokens per batch element of the k input
  // Head-sharded layer, token-scope norm: per-token sums of squares over all
  // the layer's heads ([B*Lq] for q, then [B*Lk_in] for k), or null (the
  // kernel sums the token's own channels); norm_inv_c = 1 / channels the
  // mean runs over.
  const float* ss_ext;
  float norm_inv_c;
};

struct K2Params {
  Grid g;
  const float* pooled_q;
  const float* pooled_k;
  const int* row_ptr;   // [rows + 1]
  int* col_idx;         // [nnz]
  int radius;           // window radius in blocks, < 0 when unbounded
  int topk;
  int sort_n;           // power of two >= the largest admissible set
  unsigned* clear_cnt;  // K1's split counters, zeroed here for the next K1 (n_clear entries)
  int n_clear;
  int ring_fb, slot0_fb;  // pooled k of window frame-block tk sits in ring slot (slot0_fb + tk) % ring_fb
  // Threshold reuse. thresh[row]: order bits of the row's k-th best score.
  // reuse == 0: select the top k (row_ptr / col_idx) and, if thresh is set,
  // record the thresholds. reuse == 1: keep every admissible block whose
  // score is >= the recorded threshold, in ascending order, into row r's
  // padded slot col_pad[r * pad_cap ...], its count into row_len[r].
  unsigned* thresh;
  int reuse;
  int* col_pad;
  int* row_len;
  int pad_cap;
};

// Pairs of neighbouring 64-token query blocks (same batch, head and frame
// group) that K3 computes as one 128-row tile over the union of their
// selected blocks, each entry kb | (which of the two selected it) <<
// kPairShift. A frame group's nHb x nWb block grid is cut into 2 x 2 groups
// of blocks; each group splits into two pairs either by columns (top with
// bottom) or by rows (left with right), whichever gives the smaller total
// union (the pair-union kernel decides from the selections and records each
// pair's two rows; a tie keeps columns). An odd last column pairs its blocks
// top with bottom, an odd last block row left with right, and a block left
// over in both stays single.
constexpr int kPairShift = 28;
__host__ __device__ inline int pairs_per_group(const Grid& g) {
  return 2 * (g.nHb / 2) * (g.nWb / 2) + (g.nWb % 2) * (g.nHb / 2) + (g.nHb % 2) * ((g.nWb + 1) / 2);
}
__host__ __device__ inline int64_t pair_count(const Grid& g) {
  return int64_t(g.B) * g.Hn * (g.nQB / g.bpf) * pairs_per_group(g);
}
// The rows (batch, head, query block) pair pr is chosen from. In a 2 x 2
// group: the group's four rows (top left, top right, bottom left, bottom
// right) and slot = which of the group's two pairs pr is (0 or 1). Otherwise
// the pair's own rows in r[0], r[1] (r[1] = -1 for a single block), r[2] =
// r[3] = -1 and slot = -1.
__host__ __device__ inline void pair_candidates(const Grid& g, int64_t pr, int r[4], int& slot) {
  const int pg = pairs_per_group(g);
  const int64_t per_bh = int64_t(g.nQB / g.bpf) * pg;
  const int bh = int(pr / per_bh);
  const int rem = int(pr % per_bh), tb = rem / pg;
  int k = rem % pg;
  const int base = bh * g.nQB + tb * g.bpf;
  const int in_groups = 2 * (g.nHb / 2) * (g.nWb / 2);
  r[2] = r[3] = -1;
  slot = -1;
  if (k < in_groups) {
    const int gi = k >> 1, gw = g.nWb / 2;
    const int h0 = 2 * (gi / gw), w0 = 2 * (gi % gw);
    r[0] = base + h0 * g.nWb + w0;
    r[1] = r[0] + 1;
    r[2] = r[0] + g.nWb;
    r[3] = r[2] + 1;
    slot = k & 1;
    return;
  }
  k -= in_groups;
  if (g.nWb % 2 && k < g.nHb / 2) {  // odd last column: top with bottom
    r[0] = base + 2 * k * g.nWb + g.nWb - 1;
    r[1] = r[0] + g.nWb;
    return;
  }
  if (g.nWb % 2) k -= g.nHb / 2;
  // odd last block row: left with right (the last of an odd row alone)
  const int w0 = 2 * k;
  r[0] = base + (g.nHb - 1) * g.nWb + w0;
  r[1] = w0 + 1 < g.nWb ? r[0] + 1 : -1;
}
struct PairParams {
  Grid g;
  int npairs;
  const int* row_ptr;     // the rows' selections (as K3 reads them: CSR, or padded + counts)
  const int* col_idx;
  const int* row_len;
  int pad_cap;
  int nkb;                // KV blocks per (batch, head): the range of block indices
  int* pair_col;          // [npairs][pair_cap]
  int* pair_len;          // [npairs]
  int2* pair_rows;        // [npairs] the pair's two rows (second -1: a single block)
  int pair_cap;
  // the attention's merge state of cut pairs, cleared here for the call that follows
  unsigned* merge_cnt;    // [cut][8]
  unsigned* merge_ready;  // [cut * kCutParts][8]
  int cut;                // cut_items(npairs, SMs)
};

struct K3Params {
  Grid g;
  const __nv_bfloat16* qhat;
  const __nv_bfloat16* khat;
  const __nv_bfloat16* v;   // raster [B][Lkv][C]
  __nv_bfloat16* out;       // raster [B][Lq][C]
  const int* row_ptr;
  const int* col_idx;
  float scale_log2;         // softmax scale * log2(e)
  unsigned* err;
  int ring_fb, slot0_fb;    // k^ / v of window frame-block tk sit in ring slot (slot0_fb + tk) % ring_fb
  // null: row r's blocks are col_idx[row_ptr[r] .. row_ptr[r+1]); else they
  // are col_idx[r * pad_cap ...], row_len[r] of them (threshold reuse)
  const int* row_len;
  int pad_cap;
  // 64-token blocks: the query-block pairs' union lists (PairParams)
  int npairs;
  const int* pair_col;
  const int* pair_len;
  const int2* pair_rows;
  int pair_cap;
  unsigned* work_counter;   // zero at launch (K2 clears it); K3's CTAs take work entries from it
  // The last cut_items work items (64-token pairs) are cut into up to
  // kCutParts parts of their KV tiles, each its own work entry; the last
  // part to finish merges them (merge state: cut_state, see CutState).
  int cut_items;
  unsigned* merge_cnt;      // [cut_items][8] arrivals per softmax warp slice
  unsigned* merge_ready;    // [cut_items * kCutParts][8] a part's partial result written
  float* part_buf;          // [cut_items * kCutParts][8][32 * (head_dim / 2) + 64]
  // Work items item_lo .. item_hi - 1 (rows, or query-block pairs); both 0:
  // all of them
  int item_lo, item_hi;
};

// Sizes of one configuration (lcsa_config.cu), derived without touching the
// heap or a device, so the plan path and the allocation-free path apply the
// same rules.
struct ConfigCore {
  Grid grid;
  int topk;                  // resolved budget in blocks
  int radius;                // window radius in blocks, -1 when unbounded
  int sort_n;                // power of two >= max_window (K2's candidate slots)
  int min_window, max_window;  // smallest / largest admissible set
  int64_t rows, nnz;         // CSR rows (b, h, qb) and kept blocks in all
  int heads_total;           // heads of the whole (possibly head-sharded) layer
  float scale;               // softmax scale
};
// Validate *c and fill *out. On failure, msg (if not null) receives a
// one-line reason; with msg null nothing is formatted.
lcsa_status_t resolve_config(const lcsa_config_t* c, ConfigCore* out, char* msg, size_t msg_cap);
// Budget in blocks from sparse_ratio (the topk_ratio formula, floored; a
// budget beyond 2^30 blocks is capped there and keeps every admissible block).
int budget_from_ratio(double sparse_ratio, int gh, int gw, int64_t blocks_per_frame);
// Admissible blocks of query block qb, and how many of them are kept.
int window_blocks(const ConfigCore& r, int qb);
int kept_blocks(const ConfigCore& r, int qb);

// The stateless call's block sets: every query and key block, ring = window.
inline void k1_all_blocks(K1Params& k1) {
  k1.n_qblk = k1.g.B * k1.g.nQB;
  k1.ring_fb = k1.k_in_fb = k1.g.Tkv / k1.g.bt;
  k1.k_first_fb = k1.slot0_fb = 0;
  k1.Lk_in = k1.g.Lkv;
}

// Launchers (return the launch's cudaError_t).
cudaError_t launch_rope_table(float2* table, int Tkv, int gh, int gw, int t0, int d, cudaStream_t s);
cudaError_t launch_prologue(const K1Params& p, cudaStream_t s);
// Per-token sums of squares of q ([nq][channels] bf16) then k ([nk][channels])
// into ss[nq + nk] (fp32); channels a multiple of 8, at most 2048.
cudaError_t launch_sumsq(const __nv_bfloat16* q, int64_t nq, const __nv_bfloat16* k, int64_t nk, int channels,
                         float* ss, cudaStream_t s);
size_t select_smem_bytes(int sort_n);
cudaError_t launch_select(const K2Params& p, cudaStream_t s);
cudaError_t launch_pair_union(const PairParams& p, cudaStream_t s);

// tcgen05 attention (128- or 64-token blocks, head_dim 128 or 64). Tensor
// maps: q^ / k^ as [rows][head_dim] bf16 with boxes of 64 columns x one block of rows
// (make_block_map, box_rows = tokens per block), V through its raster layout
// (make_raster_map). The kernel is persistent over min(rows, num_sms) CTAs.
bool attention_tc_supported(const Grid& g);
cudaError_t make_block_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows, int head_dim);
cudaError_t make_raster_map(CUtensorMap* map, const void* base, const Grid& g);
// q^ / k^ ([B][Hn][nblk][nb][head_dim]) seen as (channel, head, token of the
// block, block, batch) with boxes of (head_dim, Hn, bw, 1, 1): one box is one raster row of
// bw tokens with all heads, token-major in shared memory (K1's bulk stores).
cudaError_t make_xhat_row_map(CUtensorMap* map, void* base, const Grid& g, int nblk);
cudaError_t launch_exp2_selftest(const float* x, float* y, int n, cudaStream_t s);
cudaError_t launch_attention_tc(const K3Params& p, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                const CUtensorMap& tm_v, int num_sms, cudaStream_t s);

// Cut work items of the attention (64-token pairs): a persistent kernel that
// hands out whole items leaves SMs idle at the end when the item count is
// not a multiple of the SM count and the items are long, so when there are
// at least as many items as CTAs the last ctas / 2 are cut into up to
// kCutParts parts (of their KV tiles), each handed out on its own; the parts
// of an item are merged by the last of them to finish. Fewer items than CTAs
// leave no tail to even out, and are not cut.
constexpr int kCutParts = 4;
inline int cut_items(int items, int ctas) { return items >= ctas ? ctas / 2 : 0; }
// floats of part_buf for n cut items: per part and softmax warp, 32 rows x
// (head_dim / 2) of O, then the rows' maxima and sums
inline size_t part_buf_floats(int n, int head_dim) {
  return size_t(n) * kCutParts * 8 * (32 * size_t(head_dim / 2) + 64);
}

}  // namespace lcsa
