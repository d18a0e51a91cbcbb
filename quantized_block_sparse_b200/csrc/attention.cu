// attention.cu - block-sparse INT8 attention over the critical key blocks, merged with the
// linear-branch output.
//
// Method: "TurboDiffusion Demystified", section "Pillar One: Low-Bit Attention
// Acceleration - SageAttention" (Q K^T on INT8 tensor cores) and section "Pillar Two:
// Sparse-Linear Attention - SLA" (exact attention only on the selected block pairs; the
// two stack as "SageSLA").
//
// Design (sm_100a):
//   * One CTA owns a PAIR of adjacent 64-row query blocks, i.e. one 128-row tile, so every
//     tensor-core instruction is a full M = 128 tcgen05.mma. The CTA walks the union of
//     the two blocks' ascending critical lists; for a key block in only one list the other
//     half's rows are masked (their P row is 0). Adjacent query blocks share most critical
//     key blocks, which also halves the K/V traffic per query row.
//   * Warp-specialised: warp 0 issues TMA loads (Q8 pair once; per union step one INT8 K
//     tile and one bf16 V tile into a 4-stage ring), warp 1 issues tcgen05.mma (kind::i8
//     S = Q8 K8^T into one of two TMEM S buffers; kind::f16 O += P V into TMEM), warps 2-5
//     run the online softmax: one thread per query row, scores dequantised by
//     s_q * s_k * log2(e), exp2 on the SFU, P rounded to bf16 into shared memory (the A
//     operand of the P V MMA). The running max is raised only when a tile's max exceeds
//     it by more than 8 (in log2 units), so the O rescale in TMEM is rare.
//   * Epilogue: O_s = O / l, plus the linear-branch O_l, rounded once to bf16.
// Every mbarrier wait is bounded (see sm100_primitives.cuh) and never traps.
#include <climits>

#include "sagesla_internal.h"
#include "sm100_primitives.cuh"

namespace sgs {
namespace {

constexpr int kStages = 3;
constexpr int kStageBytes = 8192 + 16384;  // K8 tile + V tile
constexpr int kOffQ = 0;
constexpr int kOffStage = 16384;
constexpr int kOffBar = kOffStage + kStages * kStageBytes;
constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2 + 1;
constexpr int kAttnSmem = kOffBar + kNumBars * 8 + 16 + 1024;  // ~91 KB: two CTAs per SM
constexpr int kAttnThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;
// Columns [0, kPolyCols) of every 64-key tile take exp2 on the FMA pipe (exp2_poly), the
// rest on the SFU (ex2.approx): this balances the two pipes, the SFU alone being slower
// than the tensor core at one exponential per score.
constexpr int kPolyCols = 16;

// TMEM columns: S0 [0,64), S1 [64,128) (int32 scores of one 128x64 tile; after the
// softmax, columns [0,32) of S_b hold the bf16 P tile, two values per column), O [128,256).
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 128;

struct AttnParams {
  const float* q_scale;
  const float* k_scale;
  const int32_t* crit;
  const __nv_bfloat16* Ol;  // nullptr when there is no marginal block
  __nv_bfloat16* out;
  int* status;
  int N, nB, k_c;
};

struct UnionWalk {
  const int32_t* c0;
  const int32_t* c1;
  int n0, n1, p0, p1;
  __device__ __forceinline__ bool next(int& j, int& flags) {
    const int a = p0 < n0 ? __ldg(c0 + p0) : INT_MAX;
    const int b = p1 < n1 ? __ldg(c1 + p1) : INT_MAX;
    if (a == INT_MAX && b == INT_MAX) return false;
    j = min(a, b);
    flags = (a == j ? 1 : 0) | (b == j ? 2 : 0);
    p0 += (a == j);
    p1 += (b == j);
    return true;
  }
};

// A drain wait ignores the abort flag: it lets copies / MMAs already in flight land
// before the CTA releases its shared memory and TMEM.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, int* status) {
  int never = 0;
  mbar_wait(bar, parity, &never, status);
}

// 2^x on the FMA pipe, for x <= ~9 (scores minus the running max, in log2 units).
// Cody-Waite style range reduction x = n + f, n = rint(x), f in [-1/2, 1/2], then a
// degree-3 polynomial for 2^f fitted for minimum relative error on [-1/2, 1/2]
// (max relative error 7.5e-5, far below the bf16 rounding P receives), and 2^n added
// to the exponent field. x is clamped at -125 so the exponent stays normal; 2^-125 is
// negligible next to a row sum >= 1.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.f);
  const float t = __fadd_rn(x, 12582912.f);  // 1.5*2^23 + rint(x): rint in the low bits
  const float n = __fsub_rn(t, 12582912.f);
  const float f = __fsub_rn(x, n);
  float p = fmaf(0.0551716648042202f, f, 0.2426111400127411f);
  p = fmaf(p, f, 0.6932609677314758f);
  p = fmaf(p, f, 0.9999280571937561f);
  // (bits(t) << 23) == n << 23 (mod 2^32): the constant's low 9 bits are zero.
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Exact int32 -> fp32 for |v| < 2^22 (an INT8 dot product over 128 channels is at most
// 128*127^2 < 2^21): add the bits of 1.5*2^23, subtract 1.5*2^23 as a float.
__device__ __forceinline__ float i2f_exact(uint32_t v) {
  return __fsub_rn(__int_as_float(static_cast<int>(v) + 0x4B400000), 12582912.f);
}

// One 64-key tile of one row: P = 2^(s*sc - m) rounded to bf16 pairs in pk, returns the
// fp32 row sum of P. RAGGED masks columns >= nvalid to 0.
template <bool RAGGED>
__device__ __forceinline__ float softmax_tile(const uint32_t (&sv)[64], float sc, float negm,
                                              int nvalid, uint32_t (&pk)[32]) {
  float ps = 0.f;
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    const float x0 = fmaf(i2f_exact(sv[c]), sc, negm);
    const float x1 = fmaf(i2f_exact(sv[c + 1]), sc, negm);
    float p0 = c < kPolyCols ? exp2_poly(x0) : ex2_approx(x0);
    float p1 = c + 1 < kPolyCols ? exp2_poly(x1) : ex2_approx(x1);
    if (RAGGED) {
      p0 = c < nvalid ? p0 : 0.f;
      p1 = c + 1 < nvalid ? p1 : 0.f;
    }
    ps += p0 + p1;
    pk[c >> 1] = pack_bf16x2(p0, p1);
  }
  return ps;
}

__device__ __forceinline__ void tmem_st32_sync(uint32_t taddr, const uint32_t (&r)[32]) {
  tmem_st32(taddr, r);
  tmem_wait_st();
}

// tcgen05.mma kind::f16 with the A operand (P, M x K) read from TMEM.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate));
}

__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, AttnParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = q_full + 1;
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_full = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_full + 1);
  __shared__ int abort_flag;

  const int pr = blockIdx.x, bh = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = 2 * pr;
  const int nB = p.nB;

  UnionWalk walk;
  walk.c0 = p.crit + (static_cast<size_t>(bh) * nB + i0) * p.k_c;
  walk.c1 = walk.c0 + p.k_c;
  walk.n0 = p.k_c;
  walk.n1 = (i0 + 1 < nB) ? p.k_c : 0;
  walk.p0 = 0;
  walk.p1 = 0;

  if (tid == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(kv_full + s), 1);
      mbar_init(smem_u32(kv_empty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(s_full + b), 1);
      mbar_init(smem_u32(p_full + b), 128);
      mbar_init(smem_u32(pv_done + b), 1);
    }
    mbar_init(smem_u32(o_full), 1);
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;
  const uint32_t sQ = smem_u32(smem + kOffQ);
  const uint32_t sStage = smem_u32(smem + kOffStage);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_expect_tx(smem_u32(q_full), 16384);
      tma_load_3d(sQ, &tmQ, smem_u32(q_full), 0, i0 * 64, bh);
      tma_load_3d(sQ + 8192, &tmQ, smem_u32(q_full), 0, i0 * 64 + 64, bh);
      int t = 0, j, fl;
      bool aborted = false;
      while (walk.next(j, fl)) {
        const int s = t % kStages;
        if (t >= kStages &&
            !mbar_wait(smem_u32(kv_empty + s), ((t / kStages) - 1) & 1, &abort_flag, p.status)) {
          aborted = true;
          break;
        }
        const uint32_t dst = sStage + s * kStageBytes;
        mbar_expect_tx(smem_u32(kv_full + s), kStageBytes);
        tma_load_3d(dst, &tmK, smem_u32(kv_full + s), 0, j * 64, bh);
        tma_load_3d(dst + 8192, &tmV, smem_u32(kv_full + s), 0, j * 64, bh);
        tma_load_3d(dst + 16384, &tmV, smem_u32(kv_full + s), 64, j * 64, bh);
        ++t;
      }
      if (aborted || abort_flag) {  // let the copies in flight land before exit
        mbar_drain(smem_u32(q_full), 0, p.status);
        for (int u = max(0, t - kStages); u < t; ++u)
          mbar_drain(smem_u32(kv_full + (u % kStages)), (u / kStages) & 1, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order QK(0), QK(1), PV(0), QK(2), PV(1), ...: tcgen05.mma ops from one thread
    // execute in issue order, so QK(t) overwriting S_(t%2) (which holds P(t-2)) runs after
    // PV(t-2) has read it.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(2, 1, 0, 0, 128, 64);
      constexpr uint32_t idesc_pv = make_idesc(1, 1, 0, 1, 128, 128);
      bool ok = mbar_wait(smem_u32(q_full), 0, &abort_flag, p.status);
      auto issue_pv = [&](int u) -> bool {
        const int s = u % kStages, b = u & 1;
        if (!mbar_wait(smem_u32(p_full + b), (u >> 1) & 1, &abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t v = sStage + s * kStageBytes + 8192;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts(taddr + kColO, taddr + 64 * b + 8 * kk, make_sdesc(v + kk * 2048, 8192, 1024),
                      idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
        mma_commit(smem_u32(kv_empty + s));
        mma_commit(smem_u32(pv_done + b));
        return true;
      };
      int t = 0, j, fl;
      while (ok && walk.next(j, fl)) {
        const int s = t % kStages, b = t & 1;
        if (!mbar_wait(smem_u32(kv_full + s), (t / kStages) & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kt = sStage + s * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_i8(taddr + 64 * b, make_sdesc(sQ + kk * 32, 16, 1024), make_sdesc(kt + kk * 32, 16, 1024),
                 idesc_qk, kk > 0 ? 1u : 0u);
        mma_commit(smem_u32(s_full + b));
        if (t >= 1 && !issue_pv(t - 1)) {
          ok = false;
          break;
        }
        ++t;
      }
      if (ok && t >= 1) ok = issue_pv(t - 1);
      mma_commit(smem_u32(o_full));
      mbar_drain(smem_u32(o_full), 0, p.status);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 2-5)
    // Thread = query row r of the 128-row tile; rows 0-63 are block i0, 64-127 block i0+1,
    // so membership of a key block is uniform within each warp.
    const int wq = warp & 3;
    const int r = 32 * wq + lane;
    const int half = r >> 6;
    const int i = i0 + half;
    const int tok = i * 64 + (r & 63);
    const bool row_valid = (i < nB) && (tok < p.N);
    const float sq = (i < nB) ? p.q_scale[static_cast<size_t>(bh) * nB + i] : 0.f;
    const float* sk = p.k_scale + static_cast<size_t>(bh) * nB;
    const uint32_t lane_off = static_cast<uint32_t>(32 * wq) << 16;
    float m_run = -INFINITY, l = 0.f;
    bool ok = true;
    int t = 0, j, fl;
    while (walk.next(j, fl)) {
      const int b = t & 1;
      const bool member = (fl >> half) & 1;  // warp-uniform
      const float skj = sk[j];
      ok = mbar_wait(smem_u32(s_full + b), (t >> 1) & 1, &abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t pk[32];
      if (member) {
        uint32_t sv[64];
        tmem_ld64_sync(taddr + lane_off + 64 * b, sv);
        const bool ragged = (j == nB - 1) && (p.N - j * 64 < 64);  // CTA-uniform
        const int nvalid = ragged ? p.N - j * 64 : 64;
        int mx = static_cast<int>(sv[0]);
#pragma unroll
        for (int c = 1; c < 64; ++c)
          if (!ragged || c < nvalid) mx = max(mx, static_cast<int>(sv[c]));
        const float sc = __fmul_rn(__fmul_rn(sq, skj), kLog2e);
        const float mt = __fmul_rn(static_cast<float>(mx), sc);
        const bool raise = mt > m_run + kRescaleThreshold;
        const bool resc = raise && (m_run != -INFINITY);
        if (__any_sync(0xffffffffu, resc)) {
          // O holds P.V of earlier tiles: wait for the last issued P.V, then rescale it.
          if (t >= 1)
            ok = mbar_wait(smem_u32(pv_done + ((t - 1) & 1)), ((t - 1) >> 1) & 1, &abort_flag,
                           p.status);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = resc ? ex2_approx(m_run - mt) : 1.f;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t o[32];
            tmem_ld32_sync(taddr + lane_off + kColO + 32 * cc, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(taddr + lane_off + kColO + 32 * cc, o);
          }
          tmem_wait_st();
          if (resc) l *= alpha;
        }
        if (raise) m_run = mt;
        l += ragged ? softmax_tile<true>(sv, sc, -m_run, nvalid, pk)
                    : softmax_tile<false>(sv, sc, -m_run, 64, pk);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      tmem_st32_sync(taddr + lane_off + 64 * b, pk);
      tc_fence_before();
      mbar_arrive(smem_u32(p_full + b));
      ++t;
    }

    // ------------------------------------------------------------ epilogue
    ok = ok && mbar_wait(smem_u32(o_full), 0, &abort_flag, p.status);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok) {
      const float inv = 1.f / l;
      const __nv_bfloat16* olr =
          p.Ol ? p.Ol + (static_cast<size_t>(bh) * p.N + (row_valid ? tok : 0)) * kHeadDim : nullptr;
      __nv_bfloat16* dst = p.out + (static_cast<size_t>(bh) * p.N + (row_valid ? tok : 0)) * kHeadDim;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        tmem_ld32_sync(taddr + lane_off + kColO + 32 * cc, o);
        if (row_valid) {
          float lin[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) lin[c] = 0.f;
          if (olr) {
            const uint4* s4 = reinterpret_cast<const uint4*>(olr + 32 * cc);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const uint4 u = s4[qq];
              const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(b2[e]);
                lin[8 * qq + 2 * e] = f.x;
                lin[8 * qq + 2 * e + 1] = f.y;
              }
            }
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * cc);
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = fmaf(__uint_as_float(o[8 * qq + e]), inv, lin[8 * qq + e]);
            d4[qq] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(taddr, kTmemCols);
}

}  // namespace

cudaError_t launch_attention(const Dims& g, const int8_t* q8, const int8_t* k8,
                             const float* q_scale, const float* k_scale, const void* v,
                             const int32_t* crit, int k_c, int m, void* out, char* ws,
                             cudaStream_t st) {
  const WsLayout L = ws_layout(g);
  CUtensorMap tmQ, tmK, tmV;
  if (!make_tmap_3d(&tmQ, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kHeadDim, g.Npad, g.BH, 128, 64) ||
      !make_tmap_3d(&tmK, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kHeadDim, g.Npad, g.BH, 128, 64) ||
      !make_tmap_3d(&tmV, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kHeadDim, g.N, g.BH, 64, 64))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
  if (e != cudaSuccess) return e;
  AttnParams p;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.crit = crit;
  p.Ol = m > 0 ? reinterpret_cast<const __nv_bfloat16*>(ws + L.Ol) : nullptr;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = reinterpret_cast<int*>(ws + L.status);
  p.N = g.N;
  p.nB = g.nB;
  p.k_c = k_c;
  {
    TraceScope ts_("attn_kernel", st);
    attn_kernel<<<dim3((g.nB + 1) / 2, g.BH), kAttnThreads, kAttnSmem, st>>>(tmQ, tmK, tmV, p);
  }
  return cudaGetLastError();
}

}  // namespace sgs
