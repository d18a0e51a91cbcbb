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
//                      (bf16 operands, fp32 accumulation in TMEM), z_j = sum phi(K~_j).
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
    if (tid < 16)
      for (int jj = 0; jj < n; ++jj) T = __fadd_rn(T, buf[jj][tid]);
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
// V tile (MN-major SW128, TMA), phi(K~)^T tile (K-major SW128), raw Q and K blocks (bulk
// copies), reduction scratch and barriers.
constexpr int kPrepSmem = 4 * 16384 + 256 + 1024;

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

// The same code byte as quant_code(x, s) (rint(fl32(x/s)), clamped), without a division on
// the common path. With rs = fl32(1/s) and y = fl32(x*rs): |x/s| <= 127*(1+2^-23) because
// s = fl32(amax/127), so |y - x/s| < 1.6e-5 and |y - fl32(x/s)| < 2e-5. Unless y lies within
// 3e-5 of a half-integer, y and fl32(x/s) round to the same integer; those rare elements take
// the exact division. rint is done by adding 1.5*2^23 (exact for |y| < 2^22): the low byte
// of the sum's bit pattern is then the two's-complement code, and |rint(y)| <= 127 needs no
// clamp. Returns the byte in bits 0-7.
constexpr float kRintMagic = 12582912.f;  // 1.5 * 2^23
__device__ __forceinline__ uint32_t quant_byte(float x, float s, float rs) {
  const float y = __fmul_rn(x, rs);
  const float t = __fadd_rn(y, kRintMagic);
  const float e = __fsub_rn(__fsub_rn(t, kRintMagic), y);  // rint(y) - y, exact
  if (fabsf(e) > 0.49997f) return static_cast<uint32_t>(quant_code(x, s)) & 0xffu;
  return __float_as_uint(t) & 0xffu;
}

__device__ __forceinline__ void unpack8(const uint4 u, float (&f)[8]) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 t = __bfloat1622float2(b[e]);
    f[2 * e] = t.x;
    f[2 * e + 1] = t.y;
  }
}

// phi feeds bf16 MMA operands and the fp32 z sums, so the fast exponential (relative error
// ~2^-21, far below the bf16 rounding of phi) is enough.
__device__ __forceinline__ float phi_f32(float x) { return x > 0.f ? __fadd_rn(x, 1.f) : __expf(x); }

// One CTA per (head, 64-token block). All three input blocks are requested at once (two
// bulk copies for the raw Q and K rows, two TMA boxes for V straight into the MN-major
// 128-byte-swizzled operand tile), so a CTA keeps 48 KB in flight and three CTAs share an SM.
__global__ void __launch_bounds__(kPrepThreads, 3) prep_block_kernel(const __grid_constant__ CUtensorMap tmV,
                                                                   const __grid_constant__ CUtensorMap tmH,
                                                                   PrepParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sB = smem;          // V: 2 groups x 64 tokens x 64 e, MN-major, SW128
  unsigned char* sA = smem + 16384;  // phi(K~)^T: 128 rows (c) x 64 tokens, K-major, SW128
  const __nv_bfloat16* sQ = reinterpret_cast<const __nv_bfloat16*>(smem + 32768);  // [64][128]
  const __nv_bfloat16* sK = reinterpret_cast<const __nv_bfloat16*>(smem + 49152);  // [64][128]
  float* red = reinterpret_cast<float*>(smem + 65536);                              // [16]
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
  float mu8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mu8[e] = p.mu[bh * kHeadDim + 8 * chunk + e];
  const float mu_c = p.mu[bh * kHeadDim + (tid & 127)];
  __syncthreads();
  if (!mbar_wait(smem_u32(bar), 0, &abort_flag, p.status)) mbar_wait_inflight(smem_u32(bar), 0, p.status);

  // ---------------- Q~ = Q*c_s and K~ = K-mu: scales and INT8 codes (4 rows x 8 channels).
  // The fp32 values are recomputed from the shared-memory rows for the codes instead of
  // being held across the block reduction (the same two fp32 operations give the same bits).
  float lq = 0.f, lk = 0.f;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int r = rg + 16 * kk;
    if (r < n) {
      float fq[8], fk[8];
      unpack8(*reinterpret_cast<const uint4*>(sQ + r * kHeadDim + 8 * chunk), fq);
      unpack8(*reinterpret_cast<const uint4*>(sK + r * kHeadDim + 8 * chunk), fk);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        lq = fmaxf(lq, fabsf(__fmul_rn(fq[e], p.c_s)));
        lk = fmaxf(lk, fabsf(__fsub_rn(fk[e], mu8[e])));
      }
    }
  }
  const float2 amax = block_max2(lq, lk, red);
  const float sq = __fdiv_rn(amax.x, 127.f), sk = __fdiv_rn(amax.y, 127.f);
  // fast path only for a normal, finite reciprocal; otherwise every element divides exactly
  const float rq = __frcp_rn(sq), rk = __frcp_rn(sk);
  const bool fast = sq > 1e-30f && sk > 1e-30f && rq < 1e30f && rk < 1e30f;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int r = rg + 16 * kk;
    uint32_t cq[2] = {0u, 0u}, ck[2] = {0u, 0u};
    if (r < n) {
      float fq[8], fk[8];
      unpack8(*reinterpret_cast<const uint4*>(sQ + r * kHeadDim + 8 * chunk), fq);
      unpack8(*reinterpret_cast<const uint4*>(sK + r * kHeadDim + 8 * chunk), fk);
      if (fast) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          cq[e >> 2] |= quant_byte(__fmul_rn(fq[e], p.c_s), sq, rq) << (8 * (e & 3));
          ck[e >> 2] |= quant_byte(__fsub_rn(fk[e], mu8[e]), sk, rk) << (8 * (e & 3));
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          cq[e >> 2] |= (static_cast<uint32_t>(quant_code(__fmul_rn(fq[e], p.c_s), sq)) & 0xffu) << (8 * (e & 3));
          ck[e >> 2] |= (static_cast<uint32_t>(quant_code(__fsub_rn(fk[e], mu8[e]), sk)) & 0xffu) << (8 * (e & 3));
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

  // ---------------- block means (warps 0-3) and phi(K~)^T, z (warps 4-7), channel c
  const int c = tid & 127;
  float zacc = 0.f;
  if (tid < 128) {
    float aq = 0.f, ak = 0.f;
    for (int r = 0; r < n; ++r) {
      aq = __fadd_rn(aq, __fmul_rn(__bfloat162float(sQ[r * kHeadDim + c]), p.c_s));
      ak = __fadd_rn(ak, __fsub_rn(__bfloat162float(sK[r * kHeadDim + c]), mu_c));
    }
    p.q_bar[blk * kHeadDim + c] = __fdiv_rn(aq, static_cast<float>(n));
    p.k_bar[blk * kHeadDim + c] = __fdiv_rn(ak, static_cast<float>(n));
  } else {
    // row c of phi(K~)^T: 64 tokens, bf16, padded tokens 0
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r0 = 8 * q + 2 * e;
        const float f0 = r0 < n ? phi_f32(__fsub_rn(__bfloat162float(sK[r0 * kHeadDim + c]), mu_c)) : 0.f;
        const float f1 =
            r0 + 1 < n ? phi_f32(__fsub_rn(__bfloat162float(sK[(r0 + 1) * kHeadDim + c]), mu_c)) : 0.f;
        zacc += f0 + f1;
        w[e] = pack_bf16x2(f0, f1);
      }
      st_shared_v4(smem_u32(sA) + sw128_offset(c, q), w[0], w[1], w[2], w[3]);
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;

  if (tid == 0) {
    constexpr uint32_t idesc = make_idesc(1, 1, 0, 1, 128, 128);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t a = make_sdesc(smem_u32(sA) + kk * 32, 16, 1024);
      const uint64_t b = make_sdesc(smem_u32(sB) + kk * 2048, 8192, 1024);
      mma_bf16(taddr, a, b, idesc, kk > 0);
    }
    mma_commit(smem_u32(bar + 1));
  }
  if (!mbar_wait(smem_u32(bar + 1), 0, &abort_flag, p.status)) mbar_wait_inflight(smem_u32(bar + 1), 0, p.status);
  tc_fence_after();

  // h_j[c][e]: TMEM lane c, column e. Warps w and w+4 split the 128 columns. The bf16 rows
  // are staged over the raw Q/K rows (dead by now) as two 128-row x 64-column tiles in the
  // 128-byte-swizzled layout (conflict-free 16-byte writes) and leave by two TMA stores.
  unsigned char* sH = smem + 32768;
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
  if (tid >= 128) p.z[blk * kHeadDim + c] = zacc;
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
