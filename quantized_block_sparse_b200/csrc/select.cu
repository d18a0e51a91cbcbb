// select.cu - block logits and the critical / marginal / negligible split per query block.
//
// Method: "TurboDiffusion Demystified", section "Pillar Two: Sparse-Linear Attention -
// SLA": only the most important block interactions are computed exactly, a linear term
// covers the middle and the rest is skipped; section "Hands-On Tutorial": --sla_topk sets
// the kept fraction (0.1 -> 90% sparsity).
//
// One CTA handles R = 2*RT query-block rows of one head (two row groups of 128 threads):
//   1. l_ij = fp32 dot of the block means in a fixed order, one fused multiply-add per
//      channel (acc = 0; for c = 0..127: acc = fl32(qbar[c]*kbar[c] + acc)), so any
//      implementation following the order gets the same bits. Each thread keeps an
//      RT x 4 tile of (row, key block) accumulators as packed f32x2 pairs (fma.rn.f32x2:
//      two correctly rounded FMAs per instruction); the key means are staged
//      channel-major in shared memory, 8 channels at a time, by a double-buffered
//      cp.async pipeline; each row mean is stored twice so one load gives a (q, q) pair.
//   2. Each row's logits become order-preserving 32-bit keys. One warp per row finds the
//      k_c-th largest key T_c and the n_neg-th smallest key T_n by a most-significant-bit
//      first search over the key bits (a warp-wide count per bit, stopping as soon as the
//      count is exactly k_c). Total order: logit descending, block index ascending.
//   3. Critical: key > T_c, plus the lowest-index blocks with key == T_c up to k_c in
//      all. Negligible: key < T_n, plus the highest-index blocks with key == T_n up to
//      n_neg. The rest is marginal. A warp-ballot compaction writes both lists in
//      ascending block order and the 0/1 bf16 marginal mask row.
#include "sagesla_internal.h"
#include "sm100_primitives.cuh"

namespace sgs {
namespace {

constexpr int kSelThreads = 256;
constexpr int kGroupThreads = 128;                    // threads per row group (two groups)
constexpr int kJPerThread = 4;                        // key blocks per thread per pass
constexpr int kJPass = kGroupThreads * kJPerThread;   // 512 key blocks per pass
constexpr int kChunk = 8;                             // channels per pipeline stage
constexpr int kKStride = kJPass + 4;                  // floats per staged channel row
constexpr int kStages = kHeadDim / kChunk;            // 16 stages per pass
constexpr int kStageFloats = kChunk * kKStride;
constexpr int kRegKeysSmall = 16;                     // keys per lane held in registers
constexpr int kRegKeysLarge = 40;

__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2_rn(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

struct SelParams {
  const float* qbar;
  const float* kbar;
  int32_t* crit;
  int32_t* marg;
  __nv_bfloat16* mask;
  float* logits;
  int nB, nBk, nBp, k_c, n_neg, m;
};

// Larger logit -> larger unsigned key; -0 and +0 map to the same key. Every finite or
// infinite logit maps to a key >= 1, so 0 marks an empty slot.
__device__ __forceinline__ uint32_t order_key(float l) {
  if (l == 0.f) l = 0.f;
  const uint32_t u = __float_as_uint(l);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Stage channels [c0, c0+kChunk) of key blocks [jbase, jbase+512) channel-major: kChunk
// lanes read one block's contiguous channels, each lane writes one (channel, block) slot.
__device__ __forceinline__ void stage_kbar(const float* kb, float* dst, int jbase, int c0, int nB,
                                           int tid) {
#pragma unroll 4
  for (int t = 0; t < kJPass * kChunk / kSelThreads; ++t) {
    const int e = tid + t * kSelThreads;
    const int jj = e / kChunk, c = e % kChunk;
    if (jbase + jj < nB)
      cp_async4(smem_u32(dst + c * kKStride + jj),
                kb + static_cast<size_t>(jbase + jj) * kHeadDim + c0 + c);
  }
}

// One row's keys for the warp: slot t of lane l is block j = 32*t + l (0 when j >= nB).
// KPL > 0 keeps them in registers (nB <= 32*KPL); KPL == 0 reads shared memory.
template <int KPL>
struct RowKeys {
  uint32_t v[KPL > 0 ? KPL : 1];
  const uint32_t* kr;
  int nB, lane, nt;
  __device__ __forceinline__ void load(const uint32_t* kr_, int nB_, int nBp, int lane_) {
    kr = kr_;
    nB = nB_;
    lane = lane_;
    nt = nBp >> 5;
    if constexpr (KPL > 0) {
#pragma unroll
      for (int t = 0; t < KPL; ++t) {
        const int j = 32 * t + lane;
        v[t] = j < nB ? kr[j] : 0u;
      }
    }
  }
  __device__ __forceinline__ uint32_t at(int t) const {
    if constexpr (KPL > 0) {
      return v[t];
    } else {
      const int j = 32 * t + lane;
      return j < nB ? kr[j] : 0u;
    }
  }
};

template <int KPL, class Pred>
__device__ __forceinline__ int warp_count(const RowKeys<KPL>& K, Pred pred) {
  int c = 0;
  if constexpr (KPL > 0) {
#pragma unroll
    for (int t = 0; t < KPL; ++t) c += pred(K.v[t]) ? 1 : 0;
  } else {
    for (int t = 0; t < K.nt; ++t) c += pred(K.at(t)) ? 1 : 0;
  }
  return __reduce_add_sync(0xffffffffu, c);
}

// Classify one row and write its lists and mask row (one warp, warp-uniform control).
template <int KPL>
__device__ void classify_row(const SelParams& p, const uint32_t* kr, size_t row, int lane) {
  RowKeys<KPL> K;
  K.load(kr, p.nB, p.nBp, lane);
  const int k_c = p.k_c, n_neg = p.n_neg;

  // k_c-th largest key: the largest T with #{key >= T} >= k_c.
  uint32_t Tc = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = Tc | (1u << bit);
    const int c = warp_count(K, [cand](uint32_t x) { return x >= cand; });
    if (c >= k_c) {
      Tc = cand;
      if (c == k_c) break;  // {key >= cand} is exactly the critical set
    }
  }
  const int need_c = k_c - warp_count(K, [Tc](uint32_t x) { return x > Tc; });

  // n_neg-th smallest key, searched as the n_neg-th largest complemented key; empty
  // slots (0) are excluded by testing 1 <= key <= X as (key - 1) < X.
  uint32_t Tn = 0;
  int need_n = 0, eq_n = 0;
  if (n_neg > 0) {
    uint32_t T = 0;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit), X = ~cand;
      const int c = warp_count(K, [X](uint32_t x) { return x - 1u < X; });
      if (c >= n_neg) {
        T = cand;
        if (c == n_neg) break;
      }
    }
    Tn = ~T;
    need_n = n_neg - warp_count(K, [Tn](uint32_t x) { return x - 1u < Tn - 1u; });
    eq_n = warp_count(K, [Tn](uint32_t x) { return x == Tn; });
  }

  const unsigned lt = (1u << lane) - 1u;
  int nc = 0, nm = 0, seen_c = 0, seen_n = 0;
  auto chunk = [&](int t, uint32_t key) {
    const int j = 32 * t + lane;
    const bool valid = j < p.nB;
    const bool eqc = valid && key == Tc;
    const unsigned be = __ballot_sync(0xffffffffu, eqc);
    const bool isc = valid && (key > Tc || (eqc && seen_c + __popc(be & lt) < need_c));
    seen_c += __popc(be);
    bool isn = false;
    if (n_neg > 0) {
      const bool eqn = valid && key == Tn;
      const unsigned bn = __ballot_sync(0xffffffffu, eqn);
      isn = valid && (key < Tn || (eqn && seen_n + __popc(bn & lt) >= eq_n - need_n));
      seen_n += __popc(bn);
    }
    const bool ism = valid && !isc && !isn;
    const unsigned bc = __ballot_sync(0xffffffffu, isc);
    const unsigned bm = __ballot_sync(0xffffffffu, ism);
    // The counts are exact by construction; the bounds only keep a row inside its list.
    const int pc = nc + __popc(bc & lt), pm = nm + __popc(bm & lt);
    if (isc && pc < k_c) p.crit[row * k_c + pc] = j;
    if (ism && pm < p.m) p.marg[row * p.m + pm] = j;
    nc += __popc(bc);
    nm += __popc(bm);
    p.mask[row * p.nBp + j] = __float2bfloat16_rn(ism ? 1.f : 0.f);
  };
  if constexpr (KPL > 0) {
#pragma unroll
    for (int t = 0; t < KPL; ++t)
      if (t < K.nt) chunk(t, K.v[t]);
  } else {
    for (int t = 0; t < K.nt; ++t) chunk(t, K.at(t));
  }
}

template <int RT>
__global__ void __launch_bounds__(kSelThreads, 2) select_kernel(SelParams p) {
  constexpr int R = 2 * RT;
  extern __shared__ __align__(16) unsigned char smem[];
  float* qd = reinterpret_cast<float*>(smem);                 // [R][2*128] row means, doubled
  float* kT = qd + R * 2 * kHeadDim;                          // [2][kChunk][kKStride]
  uint32_t* keys = reinterpret_cast<uint32_t*>(kT + 2 * kStageFloats);  // [R][nBk]

  const int tid = threadIdx.x, bh = blockIdx.y;
  const int nB = p.nB, i0 = blockIdx.x * R;
  const int rows = min(R, nB - i0);
  const float* kb = p.kbar + static_cast<size_t>(bh) * nB * kHeadDim;

  for (int x = tid; x < R * kHeadDim / 2; x += kSelThreads) {
    const int r = x / (kHeadDim / 2);
    const float2 v = r < rows ? reinterpret_cast<const float2*>(p.qbar + (static_cast<size_t>(bh) * nB + i0) * kHeadDim)[x]
                              : make_float2(0.f, 0.f);
    reinterpret_cast<float4*>(qd)[x] = make_float4(v.x, v.x, v.y, v.y);
  }

  // ---- 1. logits, 512 key blocks per pass
  const int rg = tid / kGroupThreads, tl = tid % kGroupThreads;
  const int row0 = rg * RT;
  for (int jbase = 0; jbase < nB; jbase += kJPass) {
    uint64_t acc[RT][2];  // (row, key blocks j0/j0+1) and (row, j0+2/j0+3)
#pragma unroll
    for (int r = 0; r < RT; ++r) acc[r][0] = acc[r][1] = 0ull;  // +0.0f pairs
    const int j0 = jbase + kJPerThread * tl;
    const bool active = j0 < nB;

    stage_kbar(kb, kT, jbase, 0, nB, tid);
    cp_async_commit();
    for (int s = 0; s < kStages; ++s) {
      if (s + 1 < kStages) {
        stage_kbar(kb, kT + ((s + 1) & 1) * kStageFloats, jbase, (s + 1) * kChunk, nB, tid);
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      if (active) {
        const float* kt = kT + (s & 1) * kStageFloats + kJPerThread * tl;
        const float* qs = qd + row0 * 2 * kHeadDim + 2 * s * kChunk;
#pragma unroll
        for (int cc = 0; cc < kChunk; cc += 2) {
          const float4 k0 = *reinterpret_cast<const float4*>(kt + cc * kKStride);
          const float4 k1 = *reinterpret_cast<const float4*>(kt + (cc + 1) * kKStride);
          const uint64_t k0a = f2pack(k0.x, k0.y), k0b = f2pack(k0.z, k0.w);
          const uint64_t k1a = f2pack(k1.x, k1.y), k1b = f2pack(k1.z, k1.w);
#pragma unroll
          for (int r = 0; r < RT; ++r) {
            const float4 q = *reinterpret_cast<const float4*>(qs + r * 2 * kHeadDim + 2 * cc);
            const uint64_t qa = f2pack(q.x, q.y), qb = f2pack(q.z, q.w);  // (q_c, q_c), (q_c+1, q_c+1)
            acc[r][0] = fma2_rn(qa, k0a, acc[r][0]);  // channel c
            acc[r][1] = fma2_rn(qa, k0b, acc[r][1]);
            acc[r][0] = fma2_rn(qb, k1a, acc[r][0]);  // channel c + 1
            acc[r][1] = fma2_rn(qb, k1b, acc[r][1]);
          }
        }
      }
      __syncthreads();
    }

    if (active) {
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const int row = row0 + r;
        if (row < rows) {
          float l[4];
          f2unpack(acc[r][0], l[0], l[1]);
          f2unpack(acc[r][1], l[2], l[3]);
          uint4 kv;
          kv.x = order_key(l[0]);
          kv.y = j0 + 1 < nB ? order_key(l[1]) : 0u;
          kv.z = j0 + 2 < nB ? order_key(l[2]) : 0u;
          kv.w = j0 + 3 < nB ? order_key(l[3]) : 0u;
          *reinterpret_cast<uint4*>(keys + row * p.nBk + j0) = kv;
          if (p.logits) {
            float* lr = p.logits + (static_cast<size_t>(bh) * nB + i0 + row) * nB;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (j0 + e < nB) lr[j0 + e] = l[e];
          }
        }
      }
    }
  }
  __syncthreads();

  // ---- 2-3. thresholds and lists, one warp per row
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < rows; r += kSelThreads / 32) {
    const size_t row = static_cast<size_t>(bh) * nB + i0 + r;
    const uint32_t* kr = keys + r * p.nBk;
    if (p.nBp <= 32 * kRegKeysSmall)
      classify_row<kRegKeysSmall>(p, kr, row, lane);
    else if (p.nBp <= 32 * kRegKeysLarge)
      classify_row<kRegKeysLarge>(p, kr, row, lane);
    else
      classify_row<0>(p, kr, row, lane);
  }
}

template <int RT>
cudaError_t launch_rt(const Dims& g, const SelParams& p, cudaStream_t st) {
  constexpr int R = 2 * RT;
  const size_t smem = static_cast<size_t>(R) * 2 * kHeadDim * 4 +
                      static_cast<size_t>(2) * kStageFloats * 4 +
                      static_cast<size_t>(R) * p.nBk * 4;
  cudaError_t e = cudaFuncSetAttribute(select_kernel<RT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  {
    TraceScope ts_("select_kernel", st);
    select_kernel<RT><<<dim3((g.nB + R - 1) / R, g.BH), kSelThreads, smem, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const Dims& g, const float* q_bar, const float* k_bar, int k_c,
                          int n_neg, int m, int32_t* crit, int32_t* marg, void* mask,
                          float* logits, cudaStream_t st) {
  SelParams p;
  p.qbar = q_bar;
  p.kbar = k_bar;
  p.crit = crit;
  p.marg = marg;
  p.mask = static_cast<__nv_bfloat16*>(mask);
  p.logits = logits;
  p.nB = g.nB;
  p.nBk = (g.nB + 3) & ~3;
  p.nBp = g.nBp;
  p.k_c = k_c;
  p.n_neg = n_neg;
  p.m = m;
  // Rows per CTA shrink with nB so that the keys of all rows fit in shared memory
  // (R * nBk * 4 bytes <= 128 KB).
  if (g.nB <= 2048) return launch_rt<8>(g, p, st);
  if (g.nB <= 4096) return launch_rt<4>(g, p, st);
  if (g.nB <= 8192) return launch_rt<2>(g, p, st);
  return cudaErrorInvalidValue;
}

}  // namespace sgs
