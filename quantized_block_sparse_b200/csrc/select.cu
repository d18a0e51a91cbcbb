// select.cu - block logits and the critical / marginal / negligible split per query block.
//
// Method: "TurboDiffusion Demystified", section "Pillar Two: Sparse-Linear Attention -
// SLA": only the most important block interactions are computed exactly, a linear term
// covers the middle and the rest is skipped; section "Hands-On Tutorial": --sla_topk sets
// the kept fraction (0.1 -> 90% sparsity).
//
// One CTA handles R = 2*RT query-block rows of one head (two row groups of 128 threads);
// R is the largest of 22, 16, 12, 8, 4 whose keys still let two CTAs share an SM:
//   1. l_ij = fp32 dot of the block means in a fixed order, one fused multiply-add per
//      channel (acc = 0; for c = 0..127: acc = fl32(qbar[c]*kbar[c] + acc)), so any
//      implementation following the order gets the same bits. Each thread keeps an
//      RT x 4 tile of (row, key block) accumulators as packed f32x2 pairs (fma.rn.f32x2:
//      two correctly rounded FMAs per instruction); the key means are staged
//      channel-major in shared memory, 8 channels at a time: 16-byte global loads run one
//      stage ahead in registers and are transposed into two alternating slots by 4-byte
//      stores, one barrier per stage; each row mean is stored twice so one load gives a
//      (q, q) pair.
//   2. Each row's logits become order-preserving 32-bit keys. One warp per row finds the
//      k_c-th largest key T_c and the n_neg-th smallest key T_n by most-significant-bit
//      first searches over the key bits, both in one loop (one warp-wide reduction per bit
//      carries both counts), each stopping as soon as its count is exact. Total order:
//      logit descending, block index ascending.
//   3. Critical: key > T_c, plus the lowest-index blocks with key == T_c up to k_c in
//      all. Negligible: key < T_n, plus the highest-index blocks with key == T_n up to
//      n_neg. The rest is marginal. A warp-ballot compaction writes both lists in
//      ascending block order and the 0/1 bf16 marginal mask row; the per-tie ballots run
//      only when a threshold splits a run of equal keys.
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

// Channels [c0, c0+kChunk) of key blocks [jbase, jbase+512): four 16-byte global loads per
// thread (float4 f holds channels c0+4*(f%2) .. +3 of block f/2), held in registers one
// stage ahead of use; blocks at or past nB read as zeros.
__device__ __forceinline__ void load_stage(const float* kb, float4 (&v)[4], int jbase, int c0, int nB,
                                           int tid) {
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int f = tid + t * kSelThreads;
    const int jj = f >> 1, g = f & 1;
    v[t] = jbase + jj < nB
               ? __ldg(reinterpret_cast<const float4*>(kb + static_cast<size_t>(jbase + jj) * kHeadDim + c0 + 4 * g))
               : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Transpose a loaded stage into its channel-major slot with 4-byte stores: for each of the
// four channels, the 32 lanes of a warp hit 16 consecutive blocks in two channel rows whose
// bank offsets differ by 16, so every store is conflict-free.
__device__ __forceinline__ void store_stage(float* dst, const float4 (&v)[4], int tid) {
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int f = tid + t * kSelThreads;
    const int jj = f >> 1, g = f & 1;
    float* d = dst + 4 * g * kKStride + jj;
    d[0] = v[t].x;
    d[kKStride] = v[t].y;
    d[2 * kKStride] = v[t].z;
    d[3 * kKStride] = v[t].w;
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

// Two warp-wide counts in one reduction: low half #pred_lo, high half #pred_hi. A row has
// at most 8192 keys, so neither half overflows into the other.
template <int KPL, class PredLo, class PredHi>
__device__ __forceinline__ void warp_count2(const RowKeys<KPL>& K, PredLo lo, PredHi hi, int& c_lo,
                                            int& c_hi) {
  uint32_t c = 0;
  if constexpr (KPL > 0) {
#pragma unroll
    for (int t = 0; t < KPL; ++t) c += (lo(K.v[t]) ? 1u : 0u) + (hi(K.v[t]) ? 0x10000u : 0u);
  } else {
    for (int t = 0; t < K.nt; ++t) {
      const uint32_t x = K.at(t);
      c += (lo(x) ? 1u : 0u) + (hi(x) ? 0x10000u : 0u);
    }
  }
  c = __reduce_add_sync(0xffffffffu, c);
  c_lo = static_cast<int>(c & 0xffffu);
  c_hi = static_cast<int>(c >> 16);
}

// Classify one row and write its lists and mask row (one warp, warp-uniform control).
//
// T_c, the k_c-th largest key, is the largest T with #{key >= T} >= k_c. The n_neg-th
// smallest valid key is T_n = ~U for the largest U with #{1 <= key <= ~U} >= n_neg; since
// key <= ~U is key < -U (two's complement, U >= 1) and empty slots hold 0, that count is
// nB - #{key >= -U}. Both are found bit by bit from the most significant bit, in one loop
// while both are open (one reduction per bit for the two counts); a search stops as soon as
// its count is exactly its target, because then no later bit can change the split.
template <int KPL>
__device__ void classify_row(const SelParams& p, const uint32_t* kr, size_t row, int lane) {
  RowKeys<KPL> K;
  K.load(kr, p.nB, p.nBp, lane);
  const int k_c = p.k_c, n_neg = p.n_neg, nB = p.nB;

  uint32_t Tc = 0, U = 0;
  bool done_c = false, done_n = n_neg <= 0;
  int bit = 31;
  for (; bit >= 0 && !done_c && !done_n; --bit) {
    const uint32_t cc = Tc | (1u << bit), cn = U | (1u << bit), tn = 0u - cn;
    int gc, gn;
    warp_count2(K, [cc](uint32_t x) { return x >= cc; }, [tn](uint32_t x) { return x >= tn; }, gc,
                gn);
    if (gc >= k_c) {
      Tc = cc;
      done_c = gc == k_c;
    }
    if (nB - gn >= n_neg) {
      U = cn;
      done_n = nB - gn == n_neg;
    }
  }
  for (; bit >= 0 && !done_c; --bit) {
    const uint32_t cc = Tc | (1u << bit);
    const int gc = warp_count(K, [cc](uint32_t x) { return x >= cc; });
    if (gc >= k_c) {
      Tc = cc;
      done_c = gc == k_c;
    }
  }
  for (; bit >= 0 && !done_n; --bit) {
    const uint32_t cn = U | (1u << bit), tn = 0u - cn;
    const int gn = warp_count(K, [tn](uint32_t x) { return x >= tn; });
    if (nB - gn >= n_neg) {
      U = cn;
      done_n = nB - gn == n_neg;
    }
  }

  // Ties at a threshold: critical takes the lowest-index keys equal to T_c, negligible the
  // highest-index keys equal to T_n. Only a split inside a run of ties needs the ballots.
  int gt_c, eq_c;
  warp_count2(K, [Tc](uint32_t x) { return x > Tc; }, [Tc](uint32_t x) { return x == Tc; }, gt_c,
              eq_c);
  const int need_c = k_c - gt_c;
  const uint32_t Tn = ~U;
  int need_n = 0, eq_n = 0;
  if (n_neg > 0) {
    int lt_n;
    warp_count2(K, [Tn](uint32_t x) { return x - 1u < Tn - 1u; },
                [Tn](uint32_t x) { return x == Tn; }, lt_n, eq_n);
    need_n = n_neg - lt_n;
  }
  const bool split_c = need_c > 0 && need_c < eq_c;
  const bool all_c = need_c > 0 && need_c >= eq_c;
  const bool split_n = need_n > 0 && need_n < eq_n;
  const bool all_n = need_n > 0 && need_n >= eq_n;

  const unsigned lt = (1u << lane) - 1u;
  int nc = 0, nm = 0, seen_c = 0, seen_n = 0;
  auto chunk = [&](int t, uint32_t key) {
    const int j = 32 * t + lane;
    const bool valid = j < nB;
    bool isc = valid && (key > Tc || (all_c && key == Tc));
    if (split_c) {
      const bool eqc = valid && key == Tc;
      const unsigned be = __ballot_sync(0xffffffffu, eqc);
      isc = isc || (eqc && seen_c + __popc(be & lt) < need_c);
      seen_c += __popc(be);
    }
    bool isn = false;
    if (n_neg > 0) {
      isn = valid && (key < Tn || (all_n && key == Tn));
      if (split_n) {
        const bool eqn = valid && key == Tn;
        const unsigned bn = __ballot_sync(0xffffffffu, eqn);
        isn = isn || (eqn && seen_n + __popc(bn & lt) >= eq_n - need_n);
        seen_n += __popc(bn);
      }
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

  // ---- 1. logits, 512 key blocks per pass; channel stages alternate between two slots
  const int rg = tid / kGroupThreads, tl = tid % kGroupThreads;
  const int row0 = rg * RT;
  for (int jbase = 0; jbase < nB; jbase += kJPass) {
    uint64_t acc[RT][2];  // (row, key blocks j0/j0+1) and (row, j0+2/j0+3)
#pragma unroll
    for (int r = 0; r < RT; ++r) acc[r][0] = acc[r][1] = 0ull;  // +0.0f pairs
    const int j0 = jbase + kJPerThread * tl;
    const bool active = j0 < nB;

    float4 ahead[4];
    load_stage(kb, ahead, jbase, 0, nB, tid);
    for (int s = 0; s < kStages; ++s) {
      // Slot s%2 was last read at stage s-2, which every thread finished before the barrier
      // of stage s-1; the barrier below publishes the slot. Stage s+1's loads stay in flight
      // across the barrier and this stage's arithmetic.
      store_stage(kT + (s & 1) * kStageFloats, ahead, tid);
      if (s + 1 < kStages) load_stage(kb, ahead, jbase, (s + 1) * kChunk, nB, tid);
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
    }
    __syncthreads();  // every read of this pass's slots precedes the next pass's stores

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

constexpr size_t kSmemTwoPerSM = 115712;    // (228 KB per SM - 2 x 1 KB reserved) / 2
constexpr size_t kSmemOnePerSM = 232448;    // 227 KB, the per-CTA opt-in limit

size_t select_smem(int RT, int nBk) {
  const size_t R = 2 * static_cast<size_t>(RT);
  return R * 2 * kHeadDim * 4 + 2 * static_cast<size_t>(kStageFloats) * 4 + R * nBk * 4;
}

template <int RT>
cudaError_t launch_rt(const Dims& g, const SelParams& p, cudaStream_t st) {
  constexpr int R = 2 * RT;
  const size_t smem = select_smem(RT, p.nBk);
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
  // Rows per CTA: the most (2 x 11, 8, 4 or 2) that still lets two CTAs share an SM with
  // the keys of all rows in shared memory; past that, the most that fit one CTA. Every CTA
  // stages the head's whole key-mean table, so fewer, taller CTAs cost less. 12 rows were
  // measured slower than 8: four of the eight warps then classify two rows, four only one.
  for (const size_t cap : {kSmemTwoPerSM, kSmemOnePerSM}) {
    if (select_smem(11, p.nBk) <= cap) return launch_rt<11>(g, p, st);
    if (select_smem(8, p.nBk) <= cap) return launch_rt<8>(g, p, st);
    if (select_smem(4, p.nBk) <= cap) return launch_rt<4>(g, p, st);
    if (select_smem(2, p.nBk) <= cap) return launch_rt<2>(g, p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sgs
