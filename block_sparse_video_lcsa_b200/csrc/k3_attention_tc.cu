// K3 (tcgen05 form): block-sparse flash attention over the CSR list with the
// 5th-generation tensor cores, tensor memory and TMA, for 128- and 64-token
// blocks. Every product is M = 128 rows x N = 128: a KV tile is 128 keys
// (one 128-token block, or two consecutive entries of a 64-token list, an odd
// last tile repeating its entry for the softmax to mask), and a query tile is
// 128 rows (one 128-token block, or two neighbouring 64-token query blocks
// over the union of their selections, each KV block masked for the rows whose
// query block did not select it). M = 64 products, measured on this part,
// issue at the M = 128 rate for half the work (M64 N128 K16 every 64 cycles)
// and leave half of each softmax warp's TMEM lanes empty.
//
// Pages: "FlashVSR: From 17.2 FPS to 57.3 FPS at 768x1408", Rebuild sparse
// attention for Hopper: a warp-specialised producer/consumer path with TMA
// loads, block-sparse attention over a fused CSR list, FFMA-form softmax math,
// strided IO and zero-copy raster V. This kernel keeps those ideas and maps
// them onto sm_100a: accumulators live in tensor memory instead of registers,
// one thread issues the MMAs, and P goes back to tensor memory as the A
// operand of the P.V product.
//
// Persistent: one CTA per SM takes work entries from a global counter: the
// producer warp draws the next one and hands it to the other roles through a
// four-slot queue in shared memory, so CTAs that drew short entries take
// more. An entry is a work item (a row (batch, head, query block), or a pair
// of 64-token query blocks) or, for the last few pairs, one part of one (up
// to kCutParts equal shares of its KV tiles): long items handed out whole
// leave SMs idle at the end when their count is not a multiple of the SM
// count. The parts of a cut pair run on whatever CTAs drew them; the last to
// finish combines them: the others leave their part's O, row maxima and row
// sums in global memory, and the last adds all parts in part order (the
// online-softmax merge), so the result does not depend on which CTA finishes
// first. Roles (352 threads):
//   warp 0  TMA producer: Q tile of the row, then K^ / V blocks of its CSR list
//           (K^ from the block-major prologue output, V straight from the
//           raster input through a 5-D tensor map: d, head, x, y, frame).
//   warp 1  S issuer: S = Q K^T (both operands in shared memory) into a ring
//           of three TMEM S buffers, running up to three KV blocks ahead of
//           the softmax; also owns the TMEM allocation.
//   warp 2  P.V issuer: O += P V with P read from TMEM.
//           Each issuer is a converged warp (every lane waits, one lane
//           chosen by elect.sync issues), so each feeds the tensor pipe one
//           kind of product: a single thread that alternates the two kinds
//           with barrier waits in between was measured to issue at half the
//           pipe's rate, and issuing from an elected lane instead of a lane-0
//           branch measured 1.5-3.5 % faster. The two streams are ordered
//           through mbarriers: S of block j+3 waits until P.V of block j
//           (which reads P_j from the same buffer) has been issued, not until
//           it has completed. The tensor pipe runs a CTA's products in the
//           order they reach it, so P.V_j reads P_j before S_{j+3} writes
//           the buffer, and completes before it; the issuing warp's
//           tcgen05.fence::before_thread_sync, the mbarrier and the S
//           issuer's fence::after_thread_sync order the two warps' issues.
//   warps 3-10 softmax, two groups of four (one warp per TMEM lane quarter):
//           the KV tiles of the CTA's work go to the groups in turn, and a
//           group's warp handles all 128 keys of its quarter's 32 rows, so
//           the two warps of a sub-partition work on different tiles at
//           different times. The row's running maximum passes from tile to
//           tile through a slot and an mbarrier per tile parity; a tile's
//           maximum is published before its exponentials are computed, and
//           it is raised only when the block maximum exceeds it by more than
//           2^8 (exact: O and the row sums use the same stale maximum), so
//           only such a tile waits for the preceding P.V to rescale O. Each
//           group keeps its own partial row sum; the two are added once at
//           the end of the row. Online softmax in the exp2 domain (scale
//           folded into log2 e), P written to TMEM as bf16 pairs; finally each
//           thread normalises and stores 64 of its row's output channels.
//           Every fourth exponential runs on the FMA pipe (Cody-Waite
//           reduction 2^x = 2^n 2^f, |f| <= 1/2, and a degree-3 minimax
//           polynomial for 2^f fitted for this kernel, relative error below
//           7.5e-5) so the MUFU unit is not the bottleneck (the pages'
//           "FFMA-form softmax math").
// TMEM columns: S ring [0,128) [128,256) [256,384), O [384,512). P of block j
// is written back into S buffer j % 3 (bf16 pairs; keys 0-63 in its columns
// 0-31, keys 64-127 in columns 64-95, each half inside the columns its own
// thread has already read).
// Shared memory: Q 32 KB, K^ ring 2 x 32 KB, V ring 3 x 32 KB, all in the
// 128-byte swizzled layout that TMA writes and the MMA descriptors read. The
// producer fetches K^ as many blocks ahead of V as the K^ ring has stages
// (K^_{j+2} before V_j), matching
// the order in which the issuers consume them.
//
// Every wait on an mbarrier is bounded (wall-clock limit); a wait that runs
// out records LCSA device error "timeout", raises a CTA-wide abort flag and
// the kernel winds down instead of hanging.
#include <cuda.h>

#include "lcsa_internal.h"

namespace lcsa {
namespace {

constexpr int kNB = 128;                    // keys per KV tile (one 128-token block or two 64-token blocks)
constexpr int kKStages = 2;
constexpr int kVStages = 3;
// A tile (Q, K^ or V) is 128 rows x head_dim bf16, stored as head_dim / 64
// blocks of 64 columns (one 128-byte swizzle atom wide), 16 KB each.
constexpr uint32_t kHalfBytes = kNB * 64 * 2;
constexpr int kThreads = 352;
constexpr int kSoftmaxWarps = 8;
constexpr int kPolyEvery = 4;  // one pair of exponentials in kPolyEvery on the FMA pipe
constexpr int kSBufs = 3;
constexpr uint32_t kColS = 0, kColO = 384, kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
#ifdef LCSA_TEST_STALL
// test-only build (liblcsa_stalltest.so): waits give up after 100 ms, so a
// test can make one run out quickly
constexpr unsigned long long kWaitLimitNs = 100000000ull;
#else
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s
#endif

constexpr int kItemSlots = 4;  // work items handed from the producer to the other roles
constexpr int kItemReaders = 2 + kSoftmaxWarps;  // S issuer, P.V issuer, softmax warps (one arrival each)
constexpr uint32_t kXchgBytes = (2 * 128 + 2 * 2 * 128) * 4;

// Shared-memory layout for head_dim D (64 or 128): the Q tile, the K^ and V
// rings, the barrier block and the row maximum / sum exchange.
template <int D>
struct Smem {
  static constexpr uint32_t tile = kNB * D * 2;
  static constexpr uint32_t q = 0;
  static constexpr uint32_t k = q + tile;
  static constexpr uint32_t v = k + kKStages * tile;
  static constexpr uint32_t bar = v + kVStages * tile;
  static constexpr uint32_t xchg = bar + 512;
  static constexpr uint32_t bytes = xchg + kXchgBytes + 1024;  // + alignment slack
};

// 2^f on [-1/2, 1/2]: degree-3 minimax coefficients (relative error 7.49e-5),
// fitted by csrc/fit_exp2_poly.py.
constexpr float kExp2C0 = 0.9999281167984009f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.24261052906513214f;
constexpr float kExp2C3 = 0.055171314626932144f;

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[kSBufs], p_full[kSBufs];
  uint64_t pv_issued[kSBufs];  // P.V of the buffer's tile issued (one arrival per tile)
  uint64_t o_done[2];  // o_done[g & 1]: P.V number g (counted per CTA) and all before it have completed
  uint64_t o_free, mma_drain[2];
  uint64_t pair[4];  // end-of-row sum exchange between the two softmax warps of a lane quarter
  uint64_t dec[4][2];  // maximum in use after a tile published, per lane quarter and tile parity
  // dynamic work distribution: the producer takes the next work item from
  // the global counter and hands it to the other roles through item[]
  uint64_t item_full[kItemSlots], item_empty[kItemSlots];
  uint64_t never;  // test-only build: a barrier nothing arrives on
  alignas(16) int4 item[kItemSlots];  // segment: item, first tile, end tile, part | parts << 16
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 512, "barrier block");
static_assert(kSoftmaxWarps == 8 && kThreads == 96 + 32 * kSoftmaxWarps, "warp roles");

struct TcParams {
  Grid g;
  int ring_fb, slot0_fb;
  const int* row_ptr;
  const int* col_idx;
  const int* row_len;  // null, or the counts of a padded CSR (threshold reuse)
  int pad_cap;
  const int* pair_col;  // paired 64-token query blocks: union lists (entries kb | marks << kPairShift)
  const int* pair_len;
  const int2* pair_rows;  // each pair's two query blocks (second -1: a single block)
  int pair_cap;
  __nv_bfloat16* out;
  float scale_log2;
  unsigned* err;
  int rows;
  // Work entries: item i < rows - cut_items is entry i; the parts of the
  // last cut_items items (up to kCutParts each) follow, one entry per part.
  // This launch runs entries entry_lo .. entry_hi - 1 (those of its items),
  // taken from work_counter (zero at launch); a cut item's parts merge
  // through the counters, ready flags and partial-result slots.
  unsigned* work_counter;
  int entry_lo, entry_hi;
  int cut_items;
  unsigned* merge_cnt;
  unsigned* merge_ready;
  float* part_buf;
  int stall_site;          // test-only build: 0, or where the first work item stalls
};

// Selected blocks of row rr: col_idx[row_begin .. row_begin + row_count).
__device__ __forceinline__ int64_t row_begin(const TcParams& p, int rr) {
  return p.row_len ? int64_t(rr) * p.pad_cap : int64_t(p.row_ptr[rr]);
}
__device__ __forceinline__ int row_count(const TcParams& p, int rr) {
  return p.row_len ? p.row_len[rr] : p.row_ptr[rr + 1] - p.row_ptr[rr];
}

// The KV list of work item rr: a row, or (PAIR) a pair of query blocks.
template <bool PAIR>
__device__ __forceinline__ int64_t list_begin(const TcParams& p, int rr) {
  return PAIR ? int64_t(rr) * p.pair_cap : row_begin(p, rr);
}
template <bool PAIR>
__device__ __forceinline__ int list_count(const TcParams& p, int rr) {
  return PAIR ? p.pair_len[rr] : row_count(p, rr);
}
constexpr int kEntryMask = (1 << kPairShift) - 1;

// ---- PTX wrappers ---------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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

// Bounded wait for the phase of `bar` with the given parity. Returns false if
// the CTA is aborting or the wall-clock limit passed (then records the error).
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort, unsigned* err,
                                       unsigned site) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        *abort = 1;
        if (atomicCAS(err, kDevErrNone, kDevErrTimeout) == kDevErrNone) {
          err[1] = site;
          err[2] = blockIdx.x;
        }
        return false;
      }
    }
  }
}

// Flags between the CTAs that share a split work item: a release store
// after the part's slice is written, and a bounded acquire poll (returns
// false if the CTA is aborting or the limit passed, then records the error).
__device__ __forceinline__ void flag_release(unsigned* f) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(f), "r"(1u) : "memory");
}
__device__ __noinline__ bool flag_wait(const unsigned* f, volatile int* abort, unsigned* err, unsigned site) {
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 0;; ++i) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    if (v) return true;
    if ((i & 15u) == 15u) {
      if (*abort) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        *abort = 1;
        if (atomicCAS(err, kDevErrNone, kDevErrTimeout) == kDevErrNone) {
          err[1] = site;
          err[2] = blockIdx.x;
        }
        return false;
      }
    }
    __nanosleep(64);
  }
}

// Wait for an issuer's own tensor-core work to finish before the TMEM is
// freed: ignores the abort flag (that work is in flight either way) and gives
// up only at the wall-clock limit.
__device__ __noinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity) && global_ns() - t0 <= kWaitLimitNs) {
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            int c4, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, %6}], "
      "[%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
      : "memory");
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile("{\n .reg .pred p;\n elect.sync _|p, 0xffffffff;\n selp.u32 %0, 1, 0, p;\n}\n" : "=r"(pred));
  return pred != 0;
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: 128-byte swizzle, descriptor version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B,
// A K-major, B K-major (b_mn = 0) or MN-major (b_mn = 1), M = 128 or 64,
// N = 128 or 64.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t b_mn, uint32_t m = 128, uint32_t n = 128) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn << 16) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
          d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

#define LCSA_R32(a) \
  "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]), "=r"(a[8]), \
      "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]), "=r"(a[16]),   \
      "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), "=r"(a[24]),  \
      "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31])
#define LCSA_W32(a)                                                                                               \
  "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]), "r"(a[8]), "r"(a[9]), \
      "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]), "r"(a[15]), "r"(a[16]), "r"(a[17]), "r"(a[18]), \
      "r"(a[19]), "r"(a[20]), "r"(a[21]), "r"(a[22]), "r"(a[23]), "r"(a[24]), "r"(a[25]), "r"(a[26]), "r"(a[27]), \
      "r"(a[28]), "r"(a[29]), "r"(a[30]), "r"(a[31])

// 32 consecutive TMEM columns of this thread's lane (warp-collective).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : LCSA_R32(r)
      : "r"(taddr));
}
// tmem_ld32 that cannot be issued before `after` is computed (an unused asm input)
__device__ __forceinline__ void tmem_ld32_after(uint32_t taddr, uint32_t (&r)[32], float after) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : LCSA_R32(r)
      : "r"(taddr), "f"(after));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      LCSA_W32(r)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float exp2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for x <= 8 on a pair of values, packed fp32x2 arithmetic (Cody-Waite):
// n = round(x) through the 1.5 * 2^23 shifter, f = x - n, 2^f by the
// polynomial, 2^n added to the exponent field. Inputs below -125 are clamped
// (the result, < 2^-124, is negligible next to the row maximum's weight of at
// least 1).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float shifter = 12582912.0f;
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = __fadd2_rn(x, make_float2(shifter, shifter));
  const float2 n = __fadd2_rn(t, make_float2(-shifter, -shifter));
  const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), x);
  float2 q = __ffma2_rn(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
  q = __ffma2_rn(q, f, make_float2(kExp2C1, kExp2C1));
  q = __ffma2_rn(q, f, make_float2(kExp2C0, kExp2C0));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + ((__float_as_uint(t.x) - 0x4B400000u) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + ((__float_as_uint(t.y) - 0x4B400000u) << 23)));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Wait of a whole warp: every lane waits, and the warp fails as one if any
// lane gave up, so warp-collective instructions never run diverged.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort, unsigned* err,
                                          unsigned site) {
  const bool ok = mbar_wait(bar, parity, abort, err, site);
  return __all_sync(0xffffffffu, ok);
}

__global__ void exp2_selftest_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 r = exp2_poly2(make_float2(x[i], i + 1 < n ? x[i + 1] : 0.0f));
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
}

// ---- the kernel -----------------------------------------------------------

// PAIR: 64-token blocks, a work item is a pair of query blocks over the union
// of their selections; otherwise 128-token blocks, a work item is one row.
// D: head_dim (64 or 128).
template <bool PAIR, int D>
__global__ void __launch_bounds__(kThreads, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  using L = Smem<D>;
  constexpr int kHalves = D / 64;  // 64-column blocks of a tile
  Bars* bars = reinterpret_cast<Bars*>(gbase + L::bar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Grid& g = p.g;
  // rows per query tile (M of the products); tokens per query / KV block and
  // KV blocks per tile: 128-token blocks, or (PAIR) 64-token blocks with two
  // query blocks in one tile and two KV blocks per KV tile
  constexpr int QM = 128;
  constexpr int NBLK = PAIR ? 64 : QM;
  constexpr int KB = kNB / NBLK;

  auto bar = [&](uint64_t& b) { return smem_u32(&b); };
  // Segment number `it` of this CTA, as every role sees it: the producer
  // takes it (take_item, below) and publishes it in item[it % slots]; the
  // other roles read it there (one arrival per reader frees the slot). An
  // item >= p.rows ends the CTA's work.
  auto read_item = [&](int it, bool& ok) -> int4 {
    const int slot = it % kItemSlots;
    if (!(ok = warp_wait(bar(bars->item_full[slot]), (it / kItemSlots) & 1, abort, p.err, 5)))
      return make_int4(p.rows, 0, 0, 0);
    const volatile int* w = reinterpret_cast<const volatile int*>(&bars->item[slot]);
    const int4 sg = make_int4(w[0], w[1], w[2], w[3]);
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(bars->item_empty[slot]));
    return sg;
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(bars->q_full), 1);
    mbar_init(bar(bars->q_empty), 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(bars->k_full[s]), 1);
      mbar_init(bar(bars->k_empty[s]), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(bars->v_full[s]), 1);
      mbar_init(bar(bars->v_empty[s]), 1);
    }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(bar(bars->s_full[s]), 1);
      mbar_init(bar(bars->p_full[s]), kSoftmaxWarps / 2);
      mbar_init(bar(bars->pv_issued[s]), 1);
    }
    mbar_init(bar(bars->o_done[0]), 1);
    mbar_init(bar(bars->o_done[1]), 1);
    mbar_init(bar(bars->o_free), kSoftmaxWarps);
    mbar_init(bar(bars->mma_drain[0]), 1);
    mbar_init(bar(bars->mma_drain[1]), 1);
    mbar_init(bar(bars->never), 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(bar(bars->pair[s]), 64);
      mbar_init(bar(bars->dec[s][0]), 32);
      mbar_init(bar(bars->dec[s][1]), 32);
    }
    for (int s = 0; s < kItemSlots; ++s) {
      mbar_init(bar(bars->item_full[s]), 1);
      mbar_init(bar(bars->item_empty[s]), kItemReaders);
    }
    bars->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer (converged warp, lane 0 issues) ----------------
    // The row's CSR entries are fetched 32 at a time by the whole warp (one
    // coalesced load), each lane turning its entry into the k^ tile row and
    // the V box coordinates; lane 0 takes them by shuffle. The issuing lane
    // thus never waits on a dependent load or an integer division per block.
    struct Entries {
      int chunk = -1;
      int krow = 0, x0 = 0, y0 = 0, f0 = 0;
    };
    int kv = 0, row_it = 0;
    int q_issued = 0, k_issued = 0, v_issued = 0;  // tiles whose loads this warp has issued
    // The next work entry of this launch, from the global counter: a whole
    // item, or (the last cut_items items) one part of one, up to kCutParts
    // equal shares of its KV tiles (fewer for an item of fewer tiles: the
    // entries of the missing parts are skipped).
    const int whole = p.rows - p.cut_items;
    auto take_item = [&](int it, bool& ok) -> int4 {
      const int slot = it % kItemSlots;
      int4 sg = make_int4(p.rows, 0, 0, 0);
      if (it >= kItemSlots &&
          !(ok = warp_wait(bar(bars->item_empty[slot]), ((it / kItemSlots) - 1) & 1, abort, p.err, 4)))
        return sg;
      if (lane == 0) {
        for (;;) {
          const int e = p.entry_lo + int(atomicAdd(p.work_counter, 1u));
          if (e >= p.entry_hi) break;  // past this launch's entries: the end
          if (e < whole) {
            sg = make_int4(e, 0, (list_count<PAIR>(p, e) + KB - 1) / KB, 1 << 16);
            break;
          }
          const int item = whole + (e - whole) / kCutParts, part = (e - whole) % kCutParts;
          const int n = (list_count<PAIR>(p, item) + KB - 1) / KB;
          const int parts = n < kCutParts ? n : kCutParts;
          if (part >= parts) continue;
          sg = make_int4(item, part * n / parts, (part + 1) * n / parts, part | (parts << 16));
          break;
        }
        bars->item[slot] = sg;
        mbar_arrive(bar(bars->item_full[slot]));
      }
      sg.x = __shfl_sync(0xffffffffu, sg.x, 0);
      sg.y = __shfl_sync(0xffffffffu, sg.y, 0);
      sg.z = __shfl_sync(0xffffffffu, sg.z, 0);
      sg.w = __shfl_sync(0xffffffffu, sg.w, 0);
      return sg;
    };
    bool ok = true;
    for (int it = 0; ok; ++it, ++row_it) {
      const int4 sg = take_item(it, ok);
      const int rr = sg.x, t0 = sg.y;
      if (!ok || rr >= p.rows) break;
      const int64_t beg = list_begin<PAIR>(p, rr);
      const int n = list_count<PAIR>(p, rr);
      int ra = rr, rb = rr;  // the query block(s) of this work item
      if constexpr (PAIR) {
        const int2 two = p.pair_rows[rr];
        ra = two.x;
        rb = two.y < 0 ? two.x : two.y;  // a single block fills both halves; the second is not written out
      }
      const int bhh = ra / g.nQB;
      const int b = bhh / g.Hn, h = bhh % g.Hn;
      if (row_it > 0 && !(ok = warp_wait(bar(bars->q_empty), (row_it - 1) & 1, abort, p.err, 1))) break;
      if (lane == 0) {
        mbar_expect_tx(bar(bars->q_full), L::tile);
#pragma unroll
        for (int hh = 0; hh < kHalves; ++hh) {
          if constexpr (PAIR) {
            tma_load_2d(base + L::q + hh * kHalfBytes, &tm_q, hh * 64, ra * NBLK, bar(bars->q_full));
            tma_load_2d(base + L::q + hh * kHalfBytes + NBLK * 128, &tm_q, hh * 64, rb * NBLK, bar(bars->q_full));
          } else {
            tma_load_2d(base + L::q + hh * kHalfBytes, &tm_q, hh * 64, rr * QM, bar(bars->q_full));
          }
        }
      }
      __syncwarp();
      q_issued = row_it + 1;
      const int steps = sg.z - t0;  // the segment's KV tiles t0 .. sg.z - 1 of the item
      auto fill = [&](Entries& e, int chunk) {
        e.chunk = chunk;
        const int j = chunk * 32 + lane;
        if (j < n) {
          const int kb = (PAIR ? p.pair_col : p.col_idx)[beg + j] & kEntryMask;
          const int fbw = kb / g.bpf, rem = kb - fbw * g.bpf;
          int slot = p.slot0_fb + fbw;  // ring slot of its frame-block (both terms below ring_fb)
          if (slot >= p.ring_fb) slot -= p.ring_fb;
          e.krow = (bhh * g.nKB + slot * g.bpf + rem) * NBLK;
          e.x0 = (rem % g.nWb) * g.bw;
          e.y0 = (rem / g.nWb) * g.bh;
          e.f0 = b * g.Tkv + slot * g.bt;
        }
      };
      Entries ke, ve;  // cursors of the K loads (kKStages steps ahead) and of the V loads
      // entry of the selected block feeding sub-tile i of step st (the item's
      // tile t0 + st; an odd last tile repeats its block; the softmax masks
      // the copy)
      auto entry = [&](Entries& e, int st, int i) -> int {
        const int j = min((t0 + st) * KB + i, n - 1);
        if (e.chunk != (j >> 5)) fill(e, j >> 5);  // warp-uniform
        return j & 31;
      };
      auto load_k = [&](int st) -> bool {
        const int kvj = kv + st, ks = kvj % kKStages, ku = kvj / kKStages;
        if (ku > 0 && !warp_wait(bar(bars->k_empty[ks]), (ku - 1) & 1, abort, p.err, 2)) return false;
        const uint32_t kdst = base + L::k + ks * L::tile;
        if (lane == 0) mbar_expect_tx(bar(bars->k_full[ks]), L::tile);
#pragma unroll
        for (int i = 0; i < KB; ++i) {
          const int src = entry(ke, st, i);
          const int krow = __shfl_sync(0xffffffffu, ke.krow, src);
          if (lane == 0) {
#pragma unroll
            for (int hh = 0; hh < kHalves; ++hh)
              tma_load_2d(kdst + hh * kHalfBytes + i * NBLK * 128, &tm_k, hh * 64, krow, bar(bars->k_full[ks]));
          }
        }
        __syncwarp();
        k_issued = kvj + 1;
        return true;
      };
      for (int st = 0; st < kKStages && st < steps && ok; ++st) ok = load_k(st);
      for (int st = 0; st < steps && ok; ++st) {
        if (st + kKStages < steps && !(ok = load_k(st + kKStages))) break;
        const int kvj = kv + st, vs = kvj % kVStages, vu = kvj / kVStages;
        if (vu > 0 && !(ok = warp_wait(bar(bars->v_empty[vs]), (vu - 1) & 1, abort, p.err, 3))) break;
        const uint32_t vdst = base + L::v + vs * L::tile;
        if (lane == 0) mbar_expect_tx(bar(bars->v_full[vs]), L::tile);
#pragma unroll
        for (int i = 0; i < KB; ++i) {
          const int src = entry(ve, st, i);
          const int x0 = __shfl_sync(0xffffffffu, ve.x0, src), y0 = __shfl_sync(0xffffffffu, ve.y0, src);
          const int f0 = __shfl_sync(0xffffffffu, ve.f0, src);
          if (lane == 0) {
#pragma unroll
            for (int hh = 0; hh < kHalves; ++hh)
              tma_load_5d(vdst + hh * kHalfBytes + i * NBLK * 128, &tm_v, hh * 64, h, x0, y0, f0, bar(bars->v_full[vs]));
          }
        }
        __syncwarp();
        v_issued = kvj + 1;
#ifdef LCSA_TEST_STALL
        if (p.stall_site == 1 && it == 0 && st == 0) {
          // give up at once, with the work item's first loads just issued
          if (lane == 0) {
            *abort = 1;
            if (atomicCAS(p.err, kDevErrNone, kDevErrTimeout) == kDevErrNone) {
              p.err[1] = 91;
              p.err[2] = blockIdx.x;
            }
          }
          __syncwarp();
          ok = false;
          break;
        }
#endif
      }
      kv += steps;
    }
    // Every load this warp issued lands before the CTA's final barrier: on a
    // normal exit the consumers have already waited for all of them, but if
    // any role gave up, tiles issued and not yet consumed may still be in
    // flight into shared memory. The last phase of each barrier is the one to
    // wait for: a stage is reloaded only after its previous tile was
    // consumed, so that phase's completion implies the earlier ones', and no
    // later phase exists (so the parity test is unambiguous). The waits ignore
    // the abort flag and give up only at the wall-clock limit.
    if (lane == 0) {
      if (q_issued > 0) mbar_drain(bar(bars->q_full), uint32_t(q_issued - 1) & 1u);
      for (int st = 0; st < kKStages; ++st)
        if (k_issued > st) {
          const int last = (k_issued - 1) - ((k_issued - 1 - st) % kKStages);
          mbar_drain(bar(bars->k_full[st]), uint32_t(last / kKStages) & 1u);
        }
      for (int st = 0; st < kVStages; ++st)
        if (v_issued > st) {
          const int last = (v_issued - 1) - ((v_issued - 1 - st) % kVStages);
          mbar_drain(bar(bars->v_full[st]), uint32_t(last / kVStages) & 1u);
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- S issuer (converged warp, lane 0 issues) ----------------
    constexpr uint32_t id_qk = idesc_bf16(0, QM);
    int kv = 0, s_it = 0, row_it = 0;
    bool ok = true, issued = false;
    for (int it = 0; ok; ++it, ++row_it) {
      const int4 sg = read_item(it, ok);
      if (!ok || sg.x >= p.rows) break;
      const int n = sg.z - sg.y;  // KV tiles of the segment
      if (!(ok = warp_wait(bar(bars->q_full), row_it & 1, abort, p.err, 10))) break;
      for (int j = 0; j < n; ++j, ++s_it) {
        const int sb = s_it % kSBufs;
        const int kvj = kv + j, ks = kvj % kKStages;
        // buffer sb last held P of block s_it - 3: its P.V must have been
        // issued (the pipe then reads P before this S overwrites it)
        if (s_it >= kSBufs &&
            !(ok = warp_wait(bar(bars->pv_issued[sb]), ((s_it / kSBufs) - 1) & 1, abort, p.err, 11)))
          break;
        if (!(ok = warp_wait(bar(bars->k_full[ks]), (kvj / kKStages) & 1, abort, p.err, 12))) break;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t qa = base + L::q, ka = base + L::k + ks * L::tile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * (QM * 128) + (kk & 3) * 32;
            mma_ss(tmem + kColS + sb * 128, sdesc(qa + qoff, 16, 1024), sdesc(ka + koff, 16, 1024), id_qk,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(bars->s_full[sb]));
          mma_commit(bar(bars->k_empty[ks]));
          if (j == n - 1) mma_commit(bar(bars->q_empty));
        }
        __syncwarp();
        issued = true;
      }
      kv += n;
    }
    if (issued) {
      if (elect_one()) mma_commit(bar(bars->mma_drain[0]));
      __syncwarp();
      mbar_drain(bar(bars->mma_drain[0]), 0);
    }
  } else if (warp == 2) {
    // ---------------- P.V issuer (converged warp, lane 0 issues) ----------------
    constexpr uint32_t id_pv = idesc_bf16(1, QM, D);
    int kv = 0, pv_it = 0, row_it = 0;
    bool ok = true, issued = false;
    for (int it = 0; ok; ++it, ++row_it) {
      const int4 sg = read_item(it, ok);
      if (!ok || sg.x >= p.rows) break;
      const int n = sg.z - sg.y;  // KV tiles of the segment
      for (int j = 0; j < n; ++j, ++pv_it) {
        const int pb = pv_it % kSBufs;
        if (!(ok = warp_wait(bar(bars->p_full[pb]), (pv_it / kSBufs) & 1, abort, p.err, 13))) break;
        const int kvi = kv + j, vs = kvi % kVStages;
        if (!(ok = warp_wait(bar(bars->v_full[vs]), (kvi / kVStages) & 1, abort, p.err, 14))) break;
        if (j == 0 && row_it > 0 && !(ok = warp_wait(bar(bars->o_free), (row_it - 1) & 1, abort, p.err, 15)))
          break;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t va = base + L::v + vs * L::tile;
          const uint32_t pa = tmem + kColS + pb * 128;
#pragma unroll
          for (int kk = 0; kk < kNB / 16; ++kk) {
            mma_ts(tmem + kColO, pa + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8), sdesc(va + kk * 2048, kHalfBytes, 1024),
                   id_pv, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(bars->o_done[pv_it & 1]));
          mma_commit(bar(bars->v_empty[vs]));
        }
        // the products above are issued: S of tile pv_it + 3 may go into
        // this buffer (the fence orders them before the arrival)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bars->pv_issued[pb]));
        issued = true;
      }
      kv += n;
    }
    if (issued) {
      if (elect_one()) mma_commit(bar(bars->mma_drain[1]));
      __syncwarp();
      mbar_drain(bar(bars->mma_drain[1]), 0);
    }
  } else {
    // ---------------- softmax / correction / epilogue ----------------
    // The KV tiles of the CTA's work are numbered s = 0, 1, ... in order; tile
    // s goes to group s & 1 (warps 3-6 or 7-10), whose warp for TMEM lane
    // quarter sp handles all 128 keys of that quarter's 32 rows. The two
    // warps of a sub-partition thus work on different tiles at different
    // times, so one's exponentials overlap the other's other work. The row's
    // running maximum passes from tile to tile: the warp of tile s waits for
    // the maximum in use after tile s - 1 (a slot and an mbarrier per tile
    // parity), takes the block maximum, decides the maximum in use after
    // tile s (raised only if the block's exceeds it by more than 2^8: O and
    // the row sums then use the same stale maximum exactly), publishes it, and
    // only then computes the exponentials. Each group keeps its own partial
    // row sum, brought to the current maximum when it next works on the row,
    // and the two are added once at the end of the row.
    const int sp = warp & 3;                 // TMEM lane quarter of this warp
    const int grp = (warp - 3) >> 2;         // which tiles (s & 1) and, at the end, which 64 channels
    const int row_in_tile = sp * 32 + lane;  // query token of this lane's row
    const uint32_t lane_addr = tmem + (uint32_t(sp * 32) << 16);
    float* xdec = reinterpret_cast<float*>(gbase + L::xchg);  // [2 tile parity][128] maximum in use
    float* xsum = xdec + 2 * 128;                              // [2 row parity][2 group][128]
    const float c = p.scale_log2;
    int s_it = 0, xk = 0;
    bool ok = true;
    // the maximum in use after tile s has been published
    auto wait_dec = [&](int s) { return warp_wait(bar(bars->dec[sp][s & 1]), (s >> 1) & 1, abort, p.err, 26); };
    for (int it = 0; ok; ++it) {
      const int4 sg = read_item(it, ok);
      const int rr = sg.x, t0 = sg.y;
      if (!ok || rr >= p.rows) break;
      const int n_sel = list_count<PAIR>(p, rr);
      const int n = sg.z - t0;  // KV tiles of the segment: the item's t0 .. t0 + n - 1
      const int* lst = PAIR ? p.pair_col + list_begin<PAIR>(p, rr) + KB * t0 : nullptr;
      const int sel_left = n_sel - KB * t0;  // list entries from the segment's first tile on
      float m_g = -INFINITY, l = 0.f;  // this group's partial row sum, scaled by 2^-m_g
      for (int j = 0; j < n && ok; ++j, ++s_it) {
        if ((s_it & 1) != grp) continue;
        // paired 64-token blocks: keys 0-63 and 64-127 are two KV blocks and
        // this quarter's rows one query block; a block counts for these rows
        // only if their query block selected it (and exists: an odd last tile
        // repeats it)
        bool mask0 = false, mask1 = false;
        if constexpr (PAIR) {
          const int bit = sp < 2 ? 1 : 2;
          mask0 = !((__ldg(lst + KB * j) >> kPairShift) & bit);
          mask1 = KB * j + 1 >= sel_left || !((__ldg(lst + KB * j + 1) >> kPairShift) & bit);
        }
        const int sb = s_it % kSBufs;
#ifdef LCSA_TEST_STALL
        // a wait that nothing ends: it runs out after the (test) limit
        if (p.stall_site == 2 && warp == 3 && it == 0 && j == 0 &&
            !(ok = warp_wait(bar(bars->never), 0, abort, p.err, 92)))
          break;
#endif
        if (!(ok = warp_wait(bar(bars->s_full[sb]), (s_it / kSBufs) & 1, abort, p.err, 20))) break;
        tc_fence_after();
        // one 64-key half in registers at a time: both halves are read for
        // the block maximum, then half 1's exponentials come from the
        // registers and half 0 is read again (keeps the warp under its
        // register share without spills)
        uint32_t sr[2][32];
        // `after`: a value the load must wait for (an asm input), so the
        // compiler cannot issue it while the previous half is still needed
        auto load_half = [&](int hh, float after) {
          tmem_ld32_after(lane_addr + kColS + sb * 128 + hh * 64, sr[0], after);
          tmem_ld32(lane_addr + kColS + sb * 128 + hh * 64 + 32, sr[1]);
          tmem_wait_ld();
        };
        // 8 independent chains of three-input max over the half in registers
        auto half_max = [&]() {
          auto sv = [&](int e) { return __uint_as_float(sr[e >> 5][e & 31]); };
          float mk[8];
#pragma unroll
          for (int a = 0; a < 8; ++a) {
            mk[a] = fmax3(sv(a), sv(a + 8), sv(a + 16));
            mk[a] = fmax3(mk[a], sv(a + 24), sv(a + 32));
            mk[a] = fmax3(mk[a], sv(a + 40), sv(a + 48));
            mk[a] = fmaxf(mk[a], sv(a + 56));
          }
          return fmax3(fmax3(mk[0], mk[1], mk[2]), fmax3(mk[3], mk[4], mk[5]), fmaxf(mk[6], mk[7]));
        };
        float mx = -INFINITY;
        if (!mask0) {
          load_half(0, 0.f);
          mx = half_max();
        }
        if (!mask1) {
          load_half(1, mx);
          mx = fmaxf(mx, half_max());
        }
        // the maximum in use so far (tile s - 1 belongs to the other group;
        // every tile waits for it, even at a row start, which keeps the
        // barrier phases in step)
        float m_prev = -INFINITY;
        if (s_it > 0) {
          if (!(ok = wait_dec(s_it - 1))) break;
          if (j > 0) m_prev = xdec[((s_it - 1) & 1) * 128 + row_in_tile];
        }
        const float m_new = fmaxf(m_prev, mx * c);
        const bool need = m_new > m_prev + kRescaleLog2;
        const float m_used = need ? m_new : m_prev;
        xdec[(s_it & 1) * 128 + row_in_tile] = m_used;
        mbar_arrive(bar(bars->dec[sp][s_it & 1]));
        if (m_g != m_used) {
          if (l != 0.f) l *= exp2_mufu(m_g - m_used);
          m_g = m_used;
        }
        const float2 c2 = make_float2(c, c), m2 = make_float2(-m_used, -m_used);
        float2 rs2[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) rs2[a] = make_float2(0.f, 0.f);
        // half 1 (in registers unless masked), then half 0 (read again)
        uint32_t pk_prev = 0u;
#pragma unroll 1
        for (int step = 0; step < 2; ++step) {
          const int hh = 1 - step;
          uint32_t pk[32];
          if (hh == 0 ? mask0 : mask1) {
#pragma unroll
            for (int e = 0; e < 32; ++e) pk[e] = 0u;
          } else {
            if (hh == 0 && !mask1) load_half(0, __uint_as_float(pk_prev));  // (half 1 masked: half 0 still in registers)
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float2 x =
                    __ffma2_rn(make_float2(__uint_as_float(sr[q2][e]), __uint_as_float(sr[q2][e + 1])), c2, m2);
                const float2 pp = ((e >> 1) % kPolyEvery == kPolyEvery - 1)
                                      ? exp2_poly2(x)
                                      : make_float2(exp2_mufu(x.x), exp2_mufu(x.y));
                rs2[(e >> 1) & 3] = __fadd2_rn(rs2[(e >> 1) & 3], pp);
                pk[q2 * 16 + (e >> 1)] = pack_bf16(pp.x, pp.y);
              }
            }
          }
          // P of keys 64 hh .. 64 hh + 63 into columns 64 hh .. 64 hh + 31 (already read)
          tmem_st32(lane_addr + kColS + sb * 128 + hh * 64, pk);
          pk_prev = pk[31];
        }
        const float2 rsum = __fadd2_rn(__fadd2_rn(rs2[0], rs2[1]), __fadd2_rn(rs2[2], rs2[3]));
        l += rsum.x + rsum.y;
        // O is rescaled when this tile raised the maximum, once every earlier
        // P.V of the row has completed; the last of them is P.V number
        // gp = s_it - 1, and P.V gp - 2 has completed (it was issued before
        // S of this tile, which has completed, and products complete in
        // issue order), so the parity wait is unambiguous
        if (j >= 1 && __any_sync(0xffffffffu, need)) {
          const float alpha = need ? exp2_mufu(m_prev - m_used) : 1.f;
          const int gp = s_it - 1;
          if (!(ok = warp_wait(bar(bars->o_done[gp & 1]), (gp >> 1) & 1, abort, p.err, 21))) break;
          tc_fence_after();
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            uint32_t o[32];
            const uint32_t oa = lane_addr + kColO + q * 32;
            tmem_ld32(oa, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(oa, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bars->p_full[sb]));
      }
      if (!ok) break;
      // epilogue: the row's final maximum, the two groups' sums brought to it
      // and added, then each group normalises and stores 64 output channels
      const int s_last = s_it - 1;
      float m_final = m_g;
      if ((s_last & 1) != grp) {
        if (!(ok = wait_dec(s_last))) break;  // waited for again by this warp's next tile: harmless
        m_final = xdec[(s_last & 1) * 128 + row_in_tile];
      }
      if (m_g != m_final && l != 0.f) l *= exp2_mufu(m_g - m_final);
      {
        // The row's last P.V is number gp = s_last (its completion implies
        // all earlier ones). A parity wait is only unambiguous while its
        // barrier is at most one phase short of the target: o_done[gp & 1]
        // last completed for P.V gp - 2, which nothing may have waited for.
        // So P.V gp - 1 is waited for first: its barrier's previous phase,
        // P.V gp - 3, was issued before S of tile gp and so has completed
        // (this group saw S of tile gp complete, directly or through the
        // other group's published maximum), and its completion implies
        // gp - 2's.
        const int gp = s_last;
        if (gp >= 1 && !(ok = warp_wait(bar(bars->o_done[(gp - 1) & 1]), ((gp - 1) >> 1) & 1, abort, p.err, 25)))
          break;
        if (!(ok = warp_wait(bar(bars->o_done[gp & 1]), (gp >> 1) & 1, abort, p.err, 22))) break;
      }
      tc_fence_after();
      // row sums, double-buffered by row: a group can start the next row's
      // epilogue before its partner has read this row's sum
      float* xs = xsum + (xk & 1) * 256;
      xs[grp * 128 + row_in_tile] = l;
      mbar_arrive(bar(bars->pair[sp]));
      if (!(ok = warp_wait(bar(bars->pair[sp]), xk & 1, abort, p.err, 24))) break;
      ++xk;
      const float l_row = l + xs[(grp ^ 1) * 128 + row_in_tile];  // the segment's row sum at m_final
      int qrow = rr, m_tok = row_in_tile;  // query block (row) and token of this lane's row
      bool store = true;
      if constexpr (PAIR) {
        const int2 two = p.pair_rows[rr];
        qrow = sp < 2 ? two.x : two.y;
        m_tok = row_in_tile & (NBLK - 1);
        store = qrow >= 0;  // a single block's second half is a copy
        qrow = store ? qrow : two.x;
      }
      const int bhh = qrow / g.nQB, qb = qrow % g.nQB;
      const int b = bhh / g.Hn, h = bhh % g.Hn;
      const int tb = qb / g.bpf, rem = qb % g.bpf;
      const int tt = m_tok / (g.bh * g.bw), yy = (m_tok / g.bw) % g.bh, xx = m_tok % g.bw;
      const int64_t tok = (int64_t(tb * g.bt + tt) * g.gh + (rem / g.nWb) * g.bh + yy) * g.gw + (rem % g.nWb) * g.bw + xx;
      // this group's half of the row's D output channels, 32 at a time
      __nv_bfloat16* dst = p.out + (int64_t(b) * g.Lq + tok) * g.C + h * D + grp * (D / 2);
      // An item cut into parts (run by whatever CTAs drew them): each warp
      // counts its part's arrival; all but the last write their slice (this
      // warp's 32 rows x D / 2 channels of O, with the rows' maxima and sums)
      // and flag it; the last waits for those flags and combines every part,
      // in part order, into the output.
      const int parts = PAIR ? sg.w >> 16 : 1, part = sg.w & 0xFFFF;  // only pairs are cut
      const int wsl = warp - 3;  // this warp's slice
      constexpr int kSlice = 32 * (D / 2) + 64;
      const int slot0 = parts > 1 ? (rr - (p.rows - p.cut_items)) * kCutParts : 0;
      auto slot_of = [&](int j) { return slot0 + j; };
      auto slice = [&](int j) { return p.part_buf + (int64_t(slot_of(j)) * 8 + wsl) * kSlice; };
      bool last = true;
      unsigned before = 0;  // parts of this slice that arrived before this one
      if (parts > 1) {
        if (lane == 0) before = atomicAdd(p.merge_cnt + int64_t(rr - (p.rows - p.cut_items)) * 8 + wsl, 1u);
        before = __shfl_sync(0xffffffffu, before, 0);
        last = before + 1 == unsigned(parts);
      }
      if (!last) {
        float* my = slice(part);
#pragma unroll
        for (int q2 = 0; q2 < D / 64; ++q2) {
          uint32_t o[32];
          tmem_ld32(lane_addr + kColO + grp * (D / 2) + q2 * 32, o);
          tmem_wait_ld();
          // channels 4 e .. 4 e + 3 of chunk q2, lane by lane (a warp's store is 512 contiguous bytes)
          float4* d4 = reinterpret_cast<float4*>(my) + q2 * 8 * 32 + lane;
#pragma unroll
          for (int e = 0; e < 8; ++e)
            d4[e * 32] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                     __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
        }
        my[32 * (D / 2) + lane] = m_final;
        my[32 * (D / 2) + 32 + lane] = l_row;
        __threadfence();
        __syncwarp();
        bool flag = true;
#ifdef LCSA_TEST_STALL
        // the first part of the first cut pair to arrive, in slice 0, leaves
        // its flag unset: the last part's wait for it runs out
        if (p.stall_site == 3 && rr == p.rows - p.cut_items && before == 0 && wsl == 0) flag = false;
#endif
        if (lane == 0 && flag) flag_release(p.merge_ready + slot_of(part) * 8 + wsl);
      } else {
        float inv;
        if (parts > 1) {
          bool got = true;
          if (lane == 0)
            for (int j = 0; j < parts && got; ++j)
              if (j != part) got = flag_wait(p.merge_ready + slot_of(j) * 8 + wsl, abort, p.err, 27);
          if (!(ok = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0)) break;
          __threadfence();
          // the row's maximum over the parts, then the sum of their sums at it
          // (every part's values read at once: at most kCutParts of them)
          float mj[kCutParts], sj[kCutParts];
          float mx = m_final;
#pragma unroll
          for (int j = 0; j < kCutParts; ++j) {
            mj[j] = j < parts && j != part ? slice(j)[32 * (D / 2) + lane] : m_final;
            mx = fmaxf(mx, mj[j]);
          }
          float lsum = 0.f;
#pragma unroll
          for (int j = 0; j < kCutParts; ++j) {
            sj[j] = j < parts && mj[j] != -INFINITY ? exp2_mufu(mj[j] - mx) : 0.f;
            const float lj = j == part ? l_row : (j < parts ? slice(j)[32 * (D / 2) + 32 + lane] : 0.f);
            if (j < parts) lsum = j == 0 ? lj * sj[j] : fmaf(lj, sj[j], lsum);
          }
          inv = 1.0f / lsum;
#pragma unroll 1
          for (int q2 = 0; q2 < D / 64; ++q2) {
            uint32_t o[32];  // this part's O
            tmem_ld32(lane_addr + kColO + grp * (D / 2) + q2 * 32, o);
            tmem_wait_ld();
            uint4 v[4];
            uint32_t* w = reinterpret_cast<uint32_t*>(v);
            // two groups of four channels at a time: the other parts' values
            // are loaded together, then added in part order at the common maximum
            constexpr int kGroup = 2;
#pragma unroll
            for (int e0 = 0; e0 < 8; e0 += kGroup) {
              float4 x[kCutParts][kGroup];
#pragma unroll
              for (int j = 0; j < kCutParts; ++j)
#pragma unroll
                for (int e = 0; e < kGroup; ++e)
                  x[j][e] = j < parts && j != part
                                ? reinterpret_cast<const float4*>(slice(j))[(q2 * 8 + e0 + e) * 32 + lane]
                                : make_float4(__uint_as_float(o[4 * (e0 + e)]), __uint_as_float(o[4 * (e0 + e) + 1]),
                                              __uint_as_float(o[4 * (e0 + e) + 2]),
                                              __uint_as_float(o[4 * (e0 + e) + 3]));
#pragma unroll
              for (int e = 0; e < kGroup; ++e) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < kCutParts; ++j) {
                  if (j >= parts) break;
                  acc[0] = j == 0 ? x[j][e].x * sj[j] : fmaf(x[j][e].x, sj[j], acc[0]);
                  acc[1] = j == 0 ? x[j][e].y * sj[j] : fmaf(x[j][e].y, sj[j], acc[1]);
                  acc[2] = j == 0 ? x[j][e].z * sj[j] : fmaf(x[j][e].z, sj[j], acc[2]);
                  acc[3] = j == 0 ? x[j][e].w * sj[j] : fmaf(x[j][e].w, sj[j], acc[3]);
                }
                w[2 * (e0 + e)] = pack_bf16(acc[0] * inv, acc[1] * inv);
                w[2 * (e0 + e) + 1] = pack_bf16(acc[2] * inv, acc[3] * inv);
              }
            }
            uint4* d4 = reinterpret_cast<uint4*>(dst + q2 * 32);
            if (store) {
#pragma unroll
              for (int e = 0; e < 4; ++e) d4[e] = v[e];
            }
          }
        } else {
          inv = 1.0f / l_row;
#pragma unroll
          for (int q2 = 0; q2 < D / 64; ++q2) {
            uint32_t o[32];
            tmem_ld32(lane_addr + kColO + grp * (D / 2) + q2 * 32, o);
            tmem_wait_ld();
            uint4 v[4];
            uint32_t* w = reinterpret_cast<uint32_t*>(v);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              w[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
            uint4* d4 = reinterpret_cast<uint4*>(dst + q2 * 32);
            if (store) {
#pragma unroll
              for (int e = 0; e < 4; ++e) d4[e] = v[e];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bars->o_free));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// ---- host side ------------------------------------------------------------

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(f);
  }
  return fn;
}

}  // namespace

bool attention_tc_supported(const Grid& g) { return g.nb == 128 || g.nb == 64; }

cudaError_t launch_exp2_selftest(const float* x, float* y, int n, cudaStream_t s) {
  exp2_selftest_kernel<<<(n + 511) / 512, 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t make_block_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows, int head_dim) {
  EncodeTiled enc = encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {cuuint64_t(head_dim), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(head_dim) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_xhat_row_map(CUtensorMap* map, void* base, const Grid& g, int nblk) {
  EncodeTiled enc = encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t tok = cuuint64_t(g.D) * 2, blk = tok * cuuint64_t(g.nb), head = blk * cuuint64_t(nblk);
  const cuuint64_t dims[5] = {cuuint64_t(g.D), cuuint64_t(g.Hn), cuuint64_t(g.nb), cuuint64_t(nblk), cuuint64_t(g.B)};
  const cuuint64_t strides[4] = {head, tok, blk, head * cuuint64_t(g.Hn)};
  const cuuint32_t box[5] = {cuuint32_t(g.D), cuuint32_t(g.Hn), cuuint32_t(g.bw), 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_raster_map(CUtensorMap* map, const void* base, const Grid& g) {
  EncodeTiled enc = encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t row = cuuint64_t(g.C) * 2;  // bytes per token
  const cuuint64_t dims[5] = {cuuint64_t(g.D), cuuint64_t(g.Hn), cuuint64_t(g.gw), cuuint64_t(g.gh),
                              cuuint64_t(g.B) * cuuint64_t(g.Tkv)};
  const cuuint64_t strides[4] = {cuuint64_t(g.D) * 2, row, row * cuuint64_t(g.gw), row * cuuint64_t(g.gw) * g.gh};
  const cuuint32_t box[5] = {64, 1, cuuint32_t(g.bw), cuuint32_t(g.bh), cuuint32_t(g.bt)};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

#ifdef LCSA_TEST_STALL
namespace {
int g_stall_site = 0;  // consumed by the next attention launch
}
#endif

cudaError_t launch_attention_tc(const K3Params& p, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                const CUtensorMap& tm_v, int num_sms, cudaStream_t s) {
  if (!attention_tc_supported(p.g)) return cudaErrorInvalidValue;
  const bool paired = p.g.nb == 64 && p.pair_col != nullptr;
  if (p.g.nb == 64 && !paired) return cudaErrorInvalidValue;  // 64-token blocks run as query-block pairs
  if (p.g.D != 64 && p.g.D != 128) return cudaErrorInvalidValue;
  auto kern = p.g.D == 128 ? (paired ? attention_tc_kernel<true, 128> : attention_tc_kernel<false, 128>)
                           : (paired ? attention_tc_kernel<true, 64> : attention_tc_kernel<false, 64>);
  const uint32_t smem = p.g.D == 128 ? Smem<128>::bytes : Smem<64>::bytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  TcParams tp{};  // every field zero unless set below
  tp.g = p.g;
  tp.row_ptr = p.row_ptr;
  tp.row_len = p.row_len;
  tp.pad_cap = p.pad_cap;
  tp.col_idx = p.col_idx;
  tp.out = p.out;
  tp.scale_log2 = p.scale_log2;
  tp.err = p.err;
  tp.rows = paired ? p.npairs : p.g.B * p.g.Hn * p.g.nQB;
  const int item_lo = p.item_lo, item_hi = p.item_hi > 0 ? p.item_hi : tp.rows;
  if (item_lo < 0 || item_hi > tp.rows || item_lo >= item_hi) return cudaErrorInvalidValue;
  tp.work_counter = p.work_counter;
  if (!tp.work_counter) return cudaErrorInvalidValue;
  // cut items (64-token pairs only): the entries of items lo .. hi - 1
  tp.cut_items = paired ? p.cut_items : 0;
  if (tp.cut_items < 0 || tp.cut_items > tp.rows) return cudaErrorInvalidValue;
  if (tp.cut_items > 0 && (!p.merge_cnt || !p.merge_ready || !p.part_buf)) return cudaErrorInvalidValue;
  tp.merge_cnt = p.merge_cnt;
  tp.merge_ready = p.merge_ready;
  tp.part_buf = p.part_buf;
  const int whole = tp.rows - tp.cut_items;
  auto entry_of = [&](int i) { return i <= whole ? i : whole + (i - whole) * kCutParts; };
  tp.entry_lo = entry_of(item_lo);
  tp.entry_hi = entry_of(item_hi);
  tp.pair_col = p.pair_col;
  tp.pair_len = p.pair_len;
  tp.pair_rows = p.pair_rows;
  tp.pair_cap = p.pair_cap;
  tp.ring_fb = p.ring_fb;
  tp.slot0_fb = p.slot0_fb;
#ifdef LCSA_TEST_STALL
  tp.stall_site = g_stall_site;
  g_stall_site = 0;
#endif
  const int entries = tp.entry_hi - tp.entry_lo;
  const int grid = entries < num_sms ? entries : num_sms;
  kern<<<grid, kThreads, smem, s>>>(tm_q, tm_k, tm_v, tp);
  return cudaGetLastError();
}

}  // namespace lcsa

#ifdef LCSA_TEST_STALL
// Test-only build: make the next attention launch give up a wait. site 1:
// the TMA producer aborts right after issuing its first work item's loads
// (they are still in flight); site 2: a softmax warp waits on a barrier
// nothing arrives on until the (100 ms) limit; site 3 (cut 64-token pairs):
// one part of the first cut pair never flags its partial result, so the last
// part's wait for it runs out. Each records LCSA_ERR_DEVICE_TIMEOUT (error
// sites 91, 92 or the waiter's own, 27 for site 3) and the kernel winds down.
extern "C" LCSA_API void lcsa_test_arm_stall(int site) { lcsa::g_stall_site = site; }
#endif
