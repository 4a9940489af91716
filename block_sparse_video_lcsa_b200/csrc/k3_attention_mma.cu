// K3 (warp-level MMA form): block-sparse flash attention over the CSR list.
//
// Pages: "FlashVSR: From 17.2 FPS to 57.3 FPS at 768x1408", Rebuild sparse
// attention for Hopper (block-sparse attention over the CSR-selected blocks,
// strided IO, V read straight from its raster layout) and What Was Actually
// Slow (attention is the largest compute block).
//
// One CTA per (batch, head, query block) row, one warp per 16 query rows.
// K^ blocks are contiguous (written block-major by the prologue); V blocks are
// gathered from the raster input row by row. Both are double-buffered in
// shared memory with cp.async; S = Q K^T and O += P V use mma.m16n8k16 (bf16
// in, fp32 accumulate); the softmax is online, in fp32, in the exp2 domain
// with the softmax scale folded into log2(e).
//
// This is the warp-synchronous tensor-core path (the form the pages' stock
// kernel uses); the tcgen05/TMEM kernel in k3_attention_tc.cu supersedes it
// for 128-token blocks.
#include "lcsa_internal.h"

namespace lcsa {
namespace {

// byte offset of element (r, c) in a [rows][128] bf16 tile with 16-byte chunks
// XOR-swizzled by (r & 7), so ldmatrix row groups hit distinct banks
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return uint32_t(r * 256 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// raster token index of token i of block `blk` on a grid with the given frames
__device__ __forceinline__ int64_t block_token(const Grid& g, int blk, int i) {
  const int tb = blk / g.bpf, rem = blk % g.bpf;
  const int hb = rem / g.nWb, wb = rem % g.nWb;
  const int tt = i / (g.bh * g.bw), yy = (i / g.bw) % g.bh, xx = i % g.bw;
  return (int64_t(tb * g.bt + tt) * g.gh + hb * g.bh + yy) * g.gw + wb * g.bw + xx;
}

template <int NB>
__global__ void __launch_bounds__(NB * 2, 1) attention_mma_kernel(const K3Params p) {
  constexpr int kThreads = NB * 2;
  constexpr int NT = NB / 8;  // key n-tiles of 8 per KV block
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t s_base = uint32_t(__cvta_generic_to_shared(smem));
  const uint32_t sQ = s_base;
  const uint32_t sK[2] = {s_base + NB * 256, s_base + 2 * NB * 256};
  const uint32_t sV[2] = {s_base + 3 * NB * 256, s_base + 4 * NB * 256};

  const Grid& g = p.g;
  const int rr = blockIdx.x;
  const int bhh = rr / g.nQB, qb = rr % g.nQB;
  const int b = bhh / g.Hn, h = bhh % g.Hn;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int beg = p.row_ptr[rr], nsel = p.row_ptr[rr + 1] - beg;

  const __nv_bfloat16* qsrc = p.qhat + int64_t(rr) * NB * kHeadDim;
  const __nv_bfloat16* kbase = p.khat + int64_t(bhh) * g.nKB * NB * kHeadDim;
  const __nv_bfloat16* vbase = p.v + int64_t(b) * g.Lkv * g.C + h * kHeadDim;

  // each thread moves 8 of the NB*16 16-byte chunks of a tile
  auto load_contig = [&](uint32_t dst, const __nv_bfloat16* src) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int ch = tid + u * kThreads;
      const int r = ch >> 4, c = (ch & 15) * 8;
      cp_async16(dst + swz(r, c), src + r * kHeadDim + c);
    }
  };
  auto load_v = [&](uint32_t dst, int kb) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int ch = tid + u * kThreads;
      const int r = ch >> 4, c = (ch & 15) * 8;
      cp_async16(dst + swz(r, c), vbase + block_token(g, kb, r) * g.C + c);
    }
  };

  load_contig(sQ, qsrc);
  if (nsel > 0) {
    const int kb0 = p.col_idx[beg];
    load_contig(sK[0], kbase + int64_t(kb0) * NB * kHeadDim);
    load_v(sV[0], kb0);
  }
  cp_commit();

  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  uint32_t qf[8][4];
  const int row0 = warp * 16;

  for (int j = 0; j < nsel; ++j) {
    const int st = j & 1;
    if (j + 1 < nsel) {
      const int kbn = p.col_idx[beg + j + 1];
      load_contig(sK[st ^ 1], kbase + int64_t(kbn) * NB * kHeadDim);
      load_v(sV[st ^ 1], kbn);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int r = row0 + (lane & 15), c = kk * 16 + (lane >> 4) * 8;
        ldsm_x4(sQ + swz(r, c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    // S = Q K^T for this warp's 16 rows and the block's NB keys
    float s[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int n = 0; n < NT; n += 2) {
        const int key = n * 8 + (lane & 7) + ((lane >> 4) << 3);
        const int c = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK[st] + swz(key, c), b0, b1, b2, b3);
        mma_bf16(s[n], qf[kk], b0, b1);
        mma_bf16(s[n + 1], qf[kk], b2, b3);
      }
    }
    // online softmax (rows lane/4 and lane/4 + 8 of this warp)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      mx[0] = fmaxf(mx[0], fmaxf(s[n][0], s[n][1]));
      mx[1] = fmaxf(mx[1], fmaxf(s[n][2], s[n][3]));
    }
    float alpha[2], mneg[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float mnew = fmaxf(m_r[r], mx[r] * p.scale_log2);
      alpha[r] = exp2f(m_r[r] - mnew);
      m_r[r] = mnew;
      mneg[r] = -mnew;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      s[n][0] = exp2f(fmaf(s[n][0], p.scale_log2, mneg[0]));
      s[n][1] = exp2f(fmaf(s[n][1], p.scale_log2, mneg[0]));
      s[n][2] = exp2f(fmaf(s[n][2], p.scale_log2, mneg[1]));
      s[n][3] = exp2f(fmaf(s[n][3], p.scale_log2, mneg[1]));
      rs[0] += s[n][0] + s[n][1];
      rs[1] += s[n][2] + s[n][3];
    }
    l_r[0] = l_r[0] * alpha[0] + rs[0];
    l_r[1] = l_r[1] * alpha[1] + rs[1];
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      o[n][0] *= alpha[0];
      o[n][1] *= alpha[0];
      o[n][2] *= alpha[1];
      o[n][3] *= alpha[1];
    }
    // O += P V
#pragma unroll
    for (int t = 0; t < NB / 16; ++t) {
      uint32_t a[4];
      a[0] = pack_bf16(s[2 * t][0], s[2 * t][1]);
      a[1] = pack_bf16(s[2 * t][2], s[2 * t][3]);
      a[2] = pack_bf16(s[2 * t + 1][0], s[2 * t + 1][1]);
      a[3] = pack_bf16(s[2 * t + 1][2], s[2 * t + 1][3]);
#pragma unroll
      for (int n = 0; n < 16; n += 2) {
        const int mtx = lane >> 3;
        const int key = t * 16 + (lane & 7) + (mtx & 1) * 8;
        const int c = n * 8 + (mtx >> 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV[st] + swz(key, c), b0, b1, b2, b3);
        mma_bf16(o[n], a, b0, b1);
        mma_bf16(o[n + 1], a, b2, b3);
      }
    }
    __syncthreads();  // stage st is refilled in the next iteration
  }

  cp_wait<0>();
  __syncthreads();  // no copy into the Q tile may still be in flight
  // finish the row sums across the four lanes of a row, normalise, stage in
  // shared memory and write the raster output with 16-byte stores
  float inv[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
    inv[r] = l_r[r] > 0.f ? 1.0f / l_r[r] : 0.f;
  }
  const int gr = lane >> 2, gc = (lane & 3) * 2;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    const uint32_t lo = pack_bf16(o[n][0] * inv[0], o[n][1] * inv[0]);
    const uint32_t hi = pack_bf16(o[n][2] * inv[1], o[n][3] * inv[1]);
    asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(sQ + swz(row0 + gr, n * 8 + gc)), "r"(lo));
    asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(sQ + swz(row0 + gr + 8, n * 8 + gc)), "r"(hi));
  }
  __syncthreads();
  __nv_bfloat16* obase = p.out + int64_t(b) * g.Lq * g.C + h * kHeadDim;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int ch = tid + u * kThreads;
    const int r = ch >> 4, c = (ch & 15) * 8;
    uint4 val;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                 : "r"(sQ + swz(r, c)));
    *reinterpret_cast<uint4*>(obase + block_token(g, qb, r) * g.C + c) = val;
  }
}

template <int NB>
cudaError_t launch_nb(const K3Params& p, cudaStream_t s) {
  const size_t smem = size_t(5) * NB * 256;
  cudaError_t e = cudaFuncSetAttribute(attention_mma_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  const int rows = p.g.B * p.g.Hn * p.g.nQB;
  attention_mma_kernel<NB><<<rows, NB * 2, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_mma(const K3Params& p, cudaStream_t s) {
  if (p.g.nb == 128) return launch_nb<128>(p, s);
  if (p.g.nb == 64) return launch_nb<64>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace lcsa
