// select.cu - block logits and the critical / marginal / negligible split per query block.
//
// Method: "TurboDiffusion Demystified", section "Pillar Two: Sparse-Linear Attention -
// SLA": only the most important block interactions are computed exactly, a linear term
// covers the middle and the rest is skipped; section "Hands-On Tutorial": --sla_topk sets
// the kept fraction (0.1 -> 90% sparsity).
//
// One CTA handles R query-block rows of one head:
//   1. l_ij = fp32 dot of the block means in a fixed order (acc = 0; for c: acc =
//      fl32(acc + fl32(qbar[c]*kbar[c]))) - no FMA, so any implementation following the
//      order gets the same bits;
//   2. each row's (l_ij, j) pairs are encoded as 64-bit keys that order by logit
//      descending, then block index ascending, and sorted by a bitonic network in shared
//      memory;
//   3. sorted positions [0,k_c) are critical, [nB-n_neg, nB) negligible, the rest
//      marginal; a warp-ballot compaction writes both lists in ascending block order and
//      the 0/1 bf16 marginal mask row.
#include "sagesla_internal.h"
#include "sm100_primitives.cuh"

namespace sgs {
namespace {

constexpr int kSelThreads = 256;
constexpr int kSelRowsMax = 16;
constexpr int kSelKeys = 8192;  // R * nBpow keys per CTA (64 KB)

struct SelParams {
  const float* qbar;
  const float* kbar;
  int32_t* crit;
  int32_t* marg;
  __nv_bfloat16* mask;
  float* logits;
  int nB, nBpow, nBp, R, k_c, n_neg, m;
};

__device__ __forceinline__ uint64_t rank_key(float l, int j) {
  if (l == 0.f) l = 0.f;  // -0 and +0 are equal logits
  uint32_t u = __float_as_uint(l);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(u) << 32) | static_cast<uint32_t>(0xFFFFFFFFu - static_cast<uint32_t>(j));
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem);                   // [R][nBpow]
  float* qb = reinterpret_cast<float*>(keys + p.R * p.nBpow);            // [R][128]
  unsigned char* cls = reinterpret_cast<unsigned char*>(qb + p.R * kHeadDim);  // [R][nBpow]

  const int i0 = blockIdx.x * p.R, bh = blockIdx.y, tid = threadIdx.x;
  const int rows = min(p.R, p.nB - i0);
  const int nB = p.nB, nBpow = p.nBpow;

  for (int x = tid; x < rows * kHeadDim; x += kSelThreads)
    qb[x] = p.qbar[(static_cast<size_t>(bh) * nB + i0) * kHeadDim + x];
  __syncthreads();

  // ---- 1. logits
  for (int j = tid; j < nBpow; j += kSelThreads) {
    if (j < nB) {
      float acc[kSelRowsMax];
#pragma unroll
      for (int r = 0; r < kSelRowsMax; ++r) acc[r] = 0.f;
      const float4* kr = reinterpret_cast<const float4*>(p.kbar + (static_cast<size_t>(bh) * nB + j) * kHeadDim);
      for (int c4 = 0; c4 < kHeadDim / 4; ++c4) {
        const float4 kv = kr[c4];
#pragma unroll
        for (int r = 0; r < kSelRowsMax; ++r) {
          if (r < rows) {
            const float4 qv = reinterpret_cast<const float4*>(qb + r * kHeadDim)[c4];
            acc[r] = __fadd_rn(acc[r], __fmul_rn(qv.x, kv.x));
            acc[r] = __fadd_rn(acc[r], __fmul_rn(qv.y, kv.y));
            acc[r] = __fadd_rn(acc[r], __fmul_rn(qv.z, kv.z));
            acc[r] = __fadd_rn(acc[r], __fmul_rn(qv.w, kv.w));
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kSelRowsMax; ++r) {
        if (r < rows) {
          keys[r * nBpow + j] = rank_key(acc[r], j);
          if (p.logits) p.logits[(static_cast<size_t>(bh) * nB + i0 + r) * nB + j] = acc[r];
        }
      }
    } else {
      for (int r = 0; r < rows; ++r) keys[r * nBpow + j] = 0ull;  // below every real key
    }
  }
  __syncthreads();

  // ---- 2. bitonic sort, descending, every row at once (nBpow = 2^lgn)
  const int lgn = __ffs(nBpow) - 1;
  const int half = nBpow >> 1;
  for (int lk = 1; lk <= lgn; ++lk) {
    for (int lj = lk - 1; lj >= 0; --lj) {
      const int jj = 1 << lj;
      for (int x = tid; x < rows * half; x += kSelThreads) {
        const int r = x >> (lgn - 1), t = x & (half - 1);
        const int i = ((t >> lj) << (lj + 1)) | (t & (jj - 1));
        const int l = i + jj;
        uint64_t* kr = keys + r * nBpow;
        const uint64_t a = kr[i], b = kr[l];
        const bool desc = ((i >> lk) & 1) == 0;
        if (desc ? (a < b) : (a > b)) {
          kr[i] = b;
          kr[l] = a;
        }
      }
      __syncthreads();
    }
  }

  // ---- 3. classes by sorted position, then ascending compaction
  for (int r = 0; r < rows; ++r) {
    for (int pos = tid; pos < nB; pos += kSelThreads) {
      const int j = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(keys[r * nBpow + pos]));
      cls[r * nBpow + j] = pos < p.k_c ? 0 : (pos < nB - p.n_neg ? 1 : 2);
    }
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const unsigned lt = (1u << lane) - 1u;
  for (int r = warp; r < rows; r += kSelThreads / 32) {
    const size_t row = static_cast<size_t>(bh) * nB + i0 + r;
    int nc = 0, nm = 0;
    for (int base = 0; base < p.nBp; base += 32) {
      const int j = base + lane;
      const int c = j < nB ? cls[r * nBpow + j] : 3;
      const unsigned bc = __ballot_sync(0xffffffffu, c == 0);
      const unsigned bm = __ballot_sync(0xffffffffu, c == 1);
      if (c == 0) p.crit[row * p.k_c + nc + __popc(bc & lt)] = j;
      if (c == 1) p.marg[row * p.m + nm + __popc(bm & lt)] = j;
      nc += __popc(bc);
      nm += __popc(bm);
      p.mask[row * p.nBp + j] = __float2bfloat16_rn(c == 1 ? 1.f : 0.f);
    }
  }
}

}  // namespace

cudaError_t launch_select(const Dims& g, const float* q_bar, const float* k_bar, int k_c,
                          int n_neg, int m, int32_t* crit, int32_t* marg, void* mask,
                          float* logits, cudaStream_t st) {
  int nBpow = 1;
  while (nBpow < g.nB) nBpow <<= 1;
  if (nBpow < 2) nBpow = 2;
  int R = kSelKeys / nBpow;
  if (R > kSelRowsMax) R = kSelRowsMax;
  if (R < 1) return cudaErrorInvalidValue;
  SelParams p;
  p.qbar = q_bar;
  p.kbar = k_bar;
  p.crit = crit;
  p.marg = marg;
  p.mask = static_cast<__nv_bfloat16*>(mask);
  p.logits = logits;
  p.nB = g.nB;
  p.nBpow = nBpow;
  p.nBp = g.nBp;
  p.R = R;
  p.k_c = k_c;
  p.n_neg = n_neg;
  p.m = m;
  const size_t smem = static_cast<size_t>(R) * nBpow * 8 + static_cast<size_t>(R) * kHeadDim * 4 +
                      static_cast<size_t>(R) * nBpow;
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  {
    TraceScope ts_("select_kernel", st);
    select_kernel<<<dim3((g.nB + R - 1) / R, g.BH), kSelThreads, smem, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace sgs
