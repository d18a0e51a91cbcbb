// prepare.cu - K smoothing, scale folding, per-block INT8 quantization, block means and the
// per-key-block linear-attention states.
//
// Method: "TurboDiffusion Demystified", section "Pillar One: Low-Bit Attention
// Acceleration - SageAttention" (INT8 attention with smoothing against outliers) and
// section "Pillar Two: Sparse-Linear Attention - SLA" (the linear-attention states).
//
// Kernels (one pass each over the inputs, HBM bound):
//   ksum_block_kernel  per (head, block): fp32 channel sums of K, token order.
//   kmean_kernel       per head: mu = (sum of block sums in block order) / N.
//   prep_block_kernel  per (head, block): Q~ = Q*c_s and K~ = K-mu, amax -> scale ->
//                      INT8 codes, block means, and h_j = phi(K~_j)^T V_j on tcgen05
//                      (bf16 operands, phi(K~) as an MN-major A tile, fp32 accumulation
//                      in TMEM), z_j = sum phi(K~_j).
// Every decision that produces an integer (codes) or a compared bit pattern (mu, scales,
// means) uses explicitly rounded fp32 operations in a fixed order (no FMA contraction).
#include "sagesla_internal.h"
#include "sm100_primitives.cuh"

namespace sgs {
namespace {

__global__ void __launch_bounds__(64) ksum_block_kernel(const __nv_bfloat16* __restrict__ k,
                                                        float* __restrict__ part, int N, int nB) {
  const int j = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int n = min(kBlock, N - j * kBlock);
  const __nv_bfloat162* src =
      reinterpret_cast<const __nv_bfloat162*>(k + (static_cast<size_t>(bh) * N + j * kBlock) * kHeadDim) + t;
  float a0 = 0.f, a1 = 0.f;
  for (int r = 0; r < n; ++r) {
    const float2 x = __bfloat1622float2(src[r * (kHeadDim / 2)]);
    a0 = __fadd_rn(a0, x.x);
    a1 = __fadd_rn(a1, x.y);
  }
  float2* dst = reinterpret_cast<float2*>(part + (static_cast<size_t>(bh) * nB + j) * kHeadDim);
  dst[t] = make_float2(a0, a1);
}

// mu[c] = (P_0[c] + P_1[c] + ... + P_{nB-1}[c]) / N, summed in block order. One CTA per
// (head, 16-channel group): the partial sums are staged through shared memory in chunks of
// 256 blocks so the sequential adds do not wait on global-memory latency.
constexpr int kMeanChunk = 256;
__global__ void __launch_bounds__(256) kmean_kernel(const float* __restrict__ part,
                                                    float* __restrict__ mu, int N, int nB) {
  __shared__ float buf[kMeanChunk][17];
  const int bh = blockIdx.x, c0 = 16 * blockIdx.y, tid = threadIdx.x;
  const float* src = part + static_cast<size_t>(bh) * nB * kHeadDim + c0;
  float T = 0.f;
  for (int base = 0; base < nB; base += kMeanChunk) {
    const int n = min(kMeanChunk, nB - base);
    for (int x = tid; x < n * 16; x += 256)
      buf[x >> 4][x & 15] = src[static_cast<size_t>(base + (x >> 4)) * kHeadDim + (x & 15)];
    __syncthreads();
    if (tid < 16) {
      // the adds stay in block order; the shared-memory loads run ahead of them
      int jj = 0;
      for (; jj + 16 <= n; jj += 16) {
        float x[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) x[u] = buf[jj + u][tid];
#pragma unroll
        for (int u = 0; u < 16; ++u) T = __fadd_rn(T, x[u]);
      }
      for (; jj < n; ++jj) T = __fadd_rn(T, buf[jj][tid]);
    }
    __syncthreads();
  }
  if (tid < 16) mu[bh * kHeadDim + c0 + tid] = __fdiv_rn(T, static_cast<float>(N));
}

struct PrepParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* mu;
  float c_s;
  int8_t* q8;
  int8_t* k8;
  float* q_scale;
  float* k_scale;
  float* q_bar;
  float* k_bar;
  __nv_bfloat16* h;
  float* z;
  int* status;
  int N, nB, Npad;
};

constexpr int kPrepThreads = 256;
// Shared memory of one CTA (1024-byte aligned base):
//   [0, 16K)      V tile, MN-major SW128 (TMA), 2 groups of 64 e x 64 tokens
//   [16K, 32K)    phi(K~) tile in the same MN-major SW128 layout (A operand, M = channel)
//   [32K, 64K)    raw Q and K rows of the block (bulk copies), [64][128] bf16 each
//   [64K, 68K)    per-warp partial z sums [8][128]
//   then block-max scratch, two mbarriers and the TMEM address slot.
// After the MMA has read them, the V and phi tiles hold the bf16 h tile for the TMA store.
constexpr int kPrepOffZ = 65536;
constexpr int kPrepOffRed = kPrepOffZ + 8 * 128 * 4;
constexpr int kPrepSmem = kPrepOffRed + 256 + 1024;

// Block max of two values at once (Q and K amax); every thread gets both results.
__device__ __forceinline__ float2 block_max2(float a, float b, float* red) {
  for (int o = 16; o > 0; o >>= 1) {
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, o));
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    red[warp] = a;
    red[8 + warp] = b;
  }
  __syncthreads();
  float ma = red[0], mb = red[8];
#pragma unroll
  for (int w = 1; w < kPrepThreads / 32; ++w) {
    ma = fmaxf(ma, red[w]);
    mb = fmaxf(mb, red[8 + w]);
  }
  return make_float2(ma, mb);
}

__device__ __forceinline__ int quant_code(float x, float s) {
  if (!(s > 0.f)) return 0;
  int c = __float2int_rn(__fdiv_rn(x, s));  // round half to even
  return max(-127, min(127, c));
}

// ---- packed fp32 pairs: each instruction rounds both lanes exactly like its scalar form.
// A packed product that feeds an add was seen to be fused with it, so every product whose
// rounding matters before an add is taken with scalar __fmul_rn instead.
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 up2(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// A bf16 pair (low half = first element) widened to an fp32 pair: exact.
__device__ __forceinline__ uint64_t bf2_f2(uint32_t u) {
  return pk2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// INT8 codes of a pair x (already Q~ or K~ in fp32), rint(fl32(x/s)) clamped to +-127,
// without a division on the common path. With rs = fl32(1/s) and y = fl32(x*rs):
// |x/s| <= 127*(1+2^-23) because s = fl32(amax/127), so |y - x/s| < 1.6e-5 and
// |y - fl32(x/s)| < 2e-5. Unless y lies within 3e-5 of a half-integer, y and fl32(x/s) round
// to the same integer; such a pair raises `bad` and the caller redoes it by exact division.
// rint is done by adding 1.5*2^23 (exact for |y| < 2^22): the low byte of the sum's bit
// pattern is then the two's-complement code, and |rint(y)| <= 127 needs no clamp.
constexpr float kRintMagic = 12582912.f;  // 1.5 * 2^23
// The product is rounded by scalar mul.rn (never contracted into the following add).
__device__ __forceinline__ uint64_t quant_pair(uint64_t x, float rs, bool& bad) {
  const uint64_t magic2 = pk2(kRintMagic, kRintMagic);
  const float2 xf = up2(x);
  const uint64_t y = pk2(__fmul_rn(xf.x, rs), __fmul_rn(xf.y, rs));
  const uint64_t t = add2(y, magic2);
  const float2 e = up2(sub2(sub2(t, magic2), y));  // rint(y) - y, exact
  bad = bad || fabsf(e.x) > 0.49997f || fabsf(e.y) > 0.49997f;
  return t;
}
// Low bytes of the four magic sums (x0, x1, x2, x3 in two pairs) as one little-endian word.
__device__ __forceinline__ uint32_t pack_codes(uint64_t t01, uint64_t t23) {
  const uint32_t lo = __byte_perm(static_cast<uint32_t>(t01), static_cast<uint32_t>(t01 >> 32), 0x0040);
  const uint32_t hi = __byte_perm(static_cast<uint32_t>(t23), static_cast<uint32_t>(t23 >> 32), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// phi(x) = elu(x) + 1 (x + 1 for x > 0, e^x otherwise). phi feeds bf16 MMA operands and the
// fp32 z sums, so e^x = 2^(x log2 e) on the SFU (relative error ~2^-22, far below the bf16
// rounding of phi) is enough.
__device__ __forceinline__ float phi_f32(float x) {
  return x > 0.f ? __fadd_rn(x, 1.f) : ex2_approx(x * 1.4426950408889634f);
}

// One CTA per (head, 64-token block), 256 threads, three CTAs per SM. All three input
// blocks are requested at once (two bulk copies for the raw Q and K rows, two TMA boxes for
// V straight into the MN-major 128-byte-swizzled operand tile). Thread (rg, chunk) owns
// rows rg, rg+16, rg+32, rg+48 and channels 8*chunk..8*chunk+7 of both Q and K:
//   pass 1  Q~ = Q*c_s and K~ = K-mu in fp32 pairs, |.| maxima, phi(K~) written straight
//           into the A operand tile (MN-major: the token-major layout of K itself) and the
//           per-thread z sums;
//   MMA     one thread issues h_j = phi(K~_j)^T V_j (4 x K=16, fp32 in TMEM);
//   pass 2  INT8 codes from the same fp32 values, recomputed from shared memory;
//   means   warps 0-3 sum Q~ and K~ down each channel in token order (fp32 pairs);
//   store   h through TMEM -> bf16 -> the freed V/phi tiles -> two TMA stores.
__global__ void __launch_bounds__(kPrepThreads, 3) prep_block_kernel(const __grid_constant__ CUtensorMap tmV,
                                                                   const __grid_constant__ CUtensorMap tmH,
                                                                   PrepParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sB = smem;          // V: 2 groups x 64 tokens x 64 e, MN-major, SW128
  unsigned char* sA = smem + 16384;  // phi(K~): 2 groups x 64 tokens x 64 c, MN-major, SW128
  const __nv_bfloat16* sQ = reinterpret_cast<const __nv_bfloat16*>(smem + 32768);  // [64][128]
  const __nv_bfloat16* sK = reinterpret_cast<const __nv_bfloat16*>(smem + 49152);  // [64][128]
  float* zred = reinterpret_cast<float*>(smem + kPrepOffZ);                         // [8][128]
  float* red = reinterpret_cast<float*>(smem + kPrepOffRed);                        // [16]
  uint64_t* bar = reinterpret_cast<uint64_t*>(red + 16);  // [0] inputs landed, [1] MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 2);
  __shared__ int abort_flag;

  const int j = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = min(kBlock, p.N - j * kBlock);
  const size_t row0 = static_cast<size_t>(bh) * p.N + static_cast<size_t>(j) * kBlock;
  const size_t prow0 = static_cast<size_t>(bh) * p.Npad + static_cast<size_t>(j) * kBlock;
  const size_t blk = static_cast<size_t>(bh) * p.nB + j;
  const int chunk = tid & 15, rg = tid >> 4;

  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 128);
  if (tid == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(bar), 1);
    mbar_init(smem_u32(bar + 1), 1);
    fence_mbar_init();
    const uint32_t rows_bytes = static_cast<uint32_t>(n) * kHeadDim * 2;
    mbar_expect_tx(smem_u32(bar), 2 * rows_bytes + 16384);
    bulk_load(smem_u32(sQ), p.q + row0 * kHeadDim, rows_bytes, smem_u32(bar));
    bulk_load(smem_u32(sK), p.k + row0 * kHeadDim, rows_bytes, smem_u32(bar));
    tma_load_3d(smem_u32(sB), &tmV, smem_u32(bar), 0, j * kBlock, bh);
    tma_load_3d(smem_u32(sB) + 8192, &tmV, smem_u32(bar), 64, j * kBlock, bh);
  }
  uint64_t mu2[4];
  {
    const float4 m0 = *reinterpret_cast<const float4*>(p.mu + bh * kHeadDim + 8 * chunk);
    const float4 m1 = *reinterpret_cast<const float4*>(p.mu + bh * kHeadDim + 8 * chunk + 4);
    mu2[0] = pk2(m0.x, m0.y);
    mu2[1] = pk2(m0.z, m0.w);
    mu2[2] = pk2(m1.x, m1.y);
    mu2[3] = pk2(m1.z, m1.w);
  }
  const uint64_t cs2 = pk2(p.c_s, p.c_s);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;
  if (!mbar_wait(smem_u32(bar), 0, &abort_flag, p.status)) mbar_wait_inflight(smem_u32(bar), 0, p.status);

  // ---------------- pass 1: maxima, phi(K~) into the A tile, z partial sums
  const uint32_t a_base = smem_u32(sA) + (chunk >> 3) * 8192;
  float lq = 0.f, lk = 0.f;
  uint64_t z2[4] = {0, 0, 0, 0};
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int r = rg + 16 * kk;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (r < n) {
      const uint4 uq = *reinterpret_cast<const uint4*>(sQ + r * kHeadDim + 8 * chunk);
      const uint4 uk = *reinterpret_cast<const uint4*>(sK + r * kHeadDim + 8 * chunk);
      const uint32_t aq[4] = {uq.x, uq.y, uq.z, uq.w}, ak[4] = {uk.x, uk.y, uk.z, uk.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 xq = up2(mul2(bf2_f2(aq[e]), cs2));
        const uint64_t xk2 = sub2(bf2_f2(ak[e]), mu2[e]);
        const float2 xk = up2(xk2);
        lq = fmaxf(lq, fmaxf(fabsf(xq.x), fabsf(xq.y)));
        lk = fmaxf(lk, fmaxf(fabsf(xk.x), fabsf(xk.y)));
        const float f0 = phi_f32(xk.x), f1 = phi_f32(xk.y);
        z2[e] = add2(z2[e], pk2(f0, f1));
        w[e] = pack_bf16x2(f0, f1);
      }
    }
    st_shared_v4(a_base + sw128_offset(r, chunk & 7), w[0], w[1], w[2], w[3]);
  }
  fence_async_smem();
  const float2 amax = block_max2(lq, lk, red);  // also publishes the A tile
  if (tid == 0) {
    tc_fence_after();
    constexpr uint32_t idesc = make_idesc(1, 1, 1, 1, 128, 128);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t a = make_sdesc(smem_u32(sA) + kk * 2048, 8192, 1024);
      const uint64_t b = make_sdesc(smem_u32(sB) + kk * 2048, 8192, 1024);
      mma_bf16(taddr, a, b, idesc, kk > 0);
    }
    mma_commit(smem_u32(bar + 1));
  }

  // ---------------- pass 2: scales and INT8 codes
  const float sq = __fdiv_rn(amax.x, 127.f), sk = __fdiv_rn(amax.y, 127.f);
  // fast path only for a normal, finite reciprocal; otherwise every element divides exactly
  const float rq = __frcp_rn(sq), rk = __frcp_rn(sk);
  const bool fast = sq > 1e-30f && sk > 1e-30f && rq < 1e30f && rk < 1e30f;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int r = rg + 16 * kk;
    uint32_t cq[2] = {0u, 0u}, ck[2] = {0u, 0u};
    if (r < n) {
      const uint4 uq = *reinterpret_cast<const uint4*>(sQ + r * kHeadDim + 8 * chunk);
      const uint4 uk = *reinterpret_cast<const uint4*>(sK + r * kHeadDim + 8 * chunk);
      const uint32_t aq[4] = {uq.x, uq.y, uq.z, uq.w}, ak[4] = {uk.x, uk.y, uk.z, uk.w};
      uint64_t xq[4], xk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        xq[e] = mul2(bf2_f2(aq[e]), cs2);
        xk[e] = sub2(bf2_f2(ak[e]), mu2[e]);
      }
      bool bad = !fast;
      uint64_t tq[4], tk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        tq[e] = quant_pair(xq[e], rq, bad);
        tk[e] = quant_pair(xk[e], rk, bad);
      }
      if (!bad) {
        cq[0] = pack_codes(tq[0], tq[1]);
        cq[1] = pack_codes(tq[2], tq[3]);
        ck[0] = pack_codes(tk[0], tk[1]);
        ck[1] = pack_codes(tk[2], tk[3]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 a = up2(xq[e]), b = up2(xk[e]);
          cq[e >> 1] |= ((static_cast<uint32_t>(quant_code(a.x, sq)) & 0xffu) |
                         ((static_cast<uint32_t>(quant_code(a.y, sq)) & 0xffu) << 8))
                        << (16 * (e & 1));
          ck[e >> 1] |= ((static_cast<uint32_t>(quant_code(b.x, sk)) & 0xffu) |
                         ((static_cast<uint32_t>(quant_code(b.y, sk)) & 0xffu) << 8))
                        << (16 * (e & 1));
        }
      }
    }
    *reinterpret_cast<uint2*>(p.q8 + (prow0 + r) * kHeadDim + 8 * chunk) = make_uint2(cq[0], cq[1]);
    *reinterpret_cast<uint2*>(p.k8 + (prow0 + r) * kHeadDim + 8 * chunk) = make_uint2(ck[0], ck[1]);
  }
  if (tid == 0) {
    p.q_scale[blk] = sq;
    p.k_scale[blk] = sk;
  }

  // ---------------- z: rows rg and rg^1 meet across the half-warps, then over the 8 warps
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 a = up2(z2[e]);
    const float b0 = __shfl_xor_sync(0xffffffffu, a.x, 16), b1 = __shfl_xor_sync(0xffffffffu, a.y, 16);
    z2[e] = pk2(a.x + b0, a.y + b1);
  }
  if (lane < 16) {
    float4* dst = reinterpret_cast<float4*>(zred + warp * 128 + 8 * chunk);
    const float2 a = up2(z2[0]), b = up2(z2[1]), c = up2(z2[2]), d = up2(z2[3]);
    dst[0] = make_float4(a.x, a.y, b.x, b.y);
    dst[1] = make_float4(c.x, c.y, d.x, d.y);
  }

  // ---------------- block means: one channel pair per thread of warps 0-3, in token order
  if (tid < 128) {
    const bool isq = tid < 64;
    const int cp = 2 * (tid & 63);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(isq ? sQ : sK) + (cp >> 1);
    const uint64_t m2 = pk2(p.mu[bh * kHeadDim + cp], p.mu[bh * kHeadDim + cp + 1]);
    uint64_t acc = pk2(0.f, 0.f);
    if (isq) {
#pragma unroll 8
      for (int r = 0; r < n; ++r) {
        const float2 x = up2(bf2_f2(src[r * (kHeadDim / 2)]));
        acc = add2(acc, pk2(__fmul_rn(x.x, p.c_s), __fmul_rn(x.y, p.c_s)));
      }
    } else {
#pragma unroll 8
      for (int r = 0; r < n; ++r) acc = add2(acc, sub2(bf2_f2(src[r * (kHeadDim / 2)]), m2));
    }
    const float2 a = up2(acc);
    float* dst = (isq ? p.q_bar : p.k_bar) + blk * kHeadDim + cp;
    *reinterpret_cast<float2*>(dst) =
        make_float2(__fdiv_rn(a.x, static_cast<float>(n)), __fdiv_rn(a.y, static_cast<float>(n)));
  }
  __syncthreads();  // zred complete
  if (tid < 128) {
    float zs = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) zs += zred[w * 128 + tid];
    p.z[blk * kHeadDim + tid] = zs;
  }

  if (!mbar_wait(smem_u32(bar + 1), 0, &abort_flag, p.status)) mbar_wait_inflight(smem_u32(bar + 1), 0, p.status);
  tc_fence_after();

  // h_j[c][e]: TMEM lane c, column e. Warps w and w+4 split the 128 columns. The bf16 rows
  // are staged in the V and phi tiles (both read by the finished MMA) as two 128-row x
  // 64-column tiles in the 128-byte-swizzled layout and leave by two TMA stores.
  unsigned char* sH = smem;
  if (!abort_flag) {
    const int cl = 32 * (warp & 3) + lane;
    const int half = warp >> 2;
    uint32_t rr[64];
    tmem_ld64_sync(taddr + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + 64 * half, rr);
    const uint32_t tile = smem_u32(sH) + half * 16384;
#pragma unroll
    for (int q = 0; q < 8; ++q)
      st_shared_v4(tile + sw128_offset(cl, q), pack_bf16x2(__uint_as_float(rr[8 * q]), __uint_as_float(rr[8 * q + 1])),
                   pack_bf16x2(__uint_as_float(rr[8 * q + 2]), __uint_as_float(rr[8 * q + 3])),
                   pack_bf16x2(__uint_as_float(rr[8 * q + 4]), __uint_as_float(rr[8 * q + 5])),
                   pack_bf16x2(__uint_as_float(rr[8 * q + 6]), __uint_as_float(rr[8 * q + 7])));
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(taddr, 128);
  if (tid == 0 && !abort_flag) {
    tma_store_3d(&tmH, smem_u32(sH), 0, j * kHeadDim, bh);
    tma_store_3d(&tmH, smem_u32(sH) + 16384, 64, j * kHeadDim, bh);
    bulk_store_commit_wait_read();
  }
}

}  // namespace

cudaError_t launch_prepare(const Dims& g, const void* q, const void* k, const void* v,
                           float sm_scale, int8_t* q8, int8_t* k8, float* q_scale,
                           float* k_scale, float* k_mean, float* q_bar, float* k_bar, void* h,
                           float* z, char* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(g);
  float* part = reinterpret_cast<float*>(ws + L.mu_part);
  int* status = reinterpret_cast<int*>(ws + L.status);
  {
    TraceScope ts_("ksum_block_kernel", st);
    ksum_block_kernel<<<dim3(g.nB, g.BH), 64, 0, st>>>(static_cast<const __nv_bfloat16*>(k), part,
                                                     g.N, g.nB);
  }
  {
    TraceScope ts_("kmean_kernel", st);
    kmean_kernel<<<dim3(g.BH, kHeadDim / 16), 256, 0, st>>>(part, k_mean, g.N, g.nB);
  }
  CUtensorMap tmV, tmH;
  if (!make_tmap_3d(&tmV, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kHeadDim, g.N, g.BH, 64, 64) ||
      !make_tmap_3d(&tmH, h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kHeadDim,
                    static_cast<uint64_t>(g.nB) * kHeadDim, g.BH, 64, 128))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(prep_block_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kPrepSmem);
  if (e != cudaSuccess) return e;
  PrepParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.mu = k_mean;
  p.c_s = sm_scale;
  p.q8 = q8;
  p.k8 = k8;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.q_bar = q_bar;
  p.k_bar = k_bar;
  p.h = static_cast<__nv_bfloat16*>(h);
  p.z = z;
  p.status = status;
  p.N = g.N;
  p.nB = g.nB;
  p.Npad = g.Npad;
  {
    TraceScope ts_("prep_block_kernel", st);
    prep_block_kernel<<<dim3(g.nB, g.BH), kPrepThreads, kPrepSmem, st>>>(tmV, tmH, p);
  }
  return cudaGetLastError();
}

}  // namespace sgs
