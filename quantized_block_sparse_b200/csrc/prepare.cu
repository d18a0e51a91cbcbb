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
constexpr int kPrepSmem = 16384 + 16384 + 64 * 128 * 4 + 1024 + 256;

__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < kPrepThreads / 32; ++w) m = fmaxf(m, red[w]);
  return m;
}

__device__ __forceinline__ int quant_code(float x, float s) {
  if (!(s > 0.f)) return 0;
  int c = __float2int_rn(__fdiv_rn(x, s));  // round half to even
  return max(-127, min(127, c));
}

// Quantize this thread's 4 rows x 8 channels and store 8 codes per row.
__device__ __forceinline__ void store_codes(const float (&x)[4][8], float s, int8_t* dst_rows,
                                            int rg, int chunk) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int r = rg + 16 * kk;
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      lo |= (static_cast<uint32_t>(quant_code(x[kk][e], s)) & 0xffu) << (8 * e);
      hi |= (static_cast<uint32_t>(quant_code(x[kk][e + 4], s)) & 0xffu) << (8 * e);
    }
    *reinterpret_cast<uint2*>(dst_rows + r * kHeadDim + 8 * chunk) = make_uint2(lo, hi);
  }
}

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 t = __bfloat1622float2(b[e]);
    f[2 * e] = t.x;
    f[2 * e + 1] = t.y;
  }
}

__device__ __forceinline__ float phi_f32(float x) { return x > 0.f ? __fadd_rn(x, 1.f) : expf(x); }

__global__ void __launch_bounds__(kPrepThreads) prep_block_kernel(PrepParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sA = smem;          // phi(K~)^T: 128 rows (c) x 64 tokens, K-major, SW128
  unsigned char* sB = smem + 16384;  // V: 2 groups x 64 tokens x 64 e, MN-major, SW128
  float* xs = reinterpret_cast<float*>(smem + 32768);  // [64][128] fp32 staging
  float* red = xs + 64 * 128;                          // [8]
  uint64_t* bar = reinterpret_cast<uint64_t*>(red + 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
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
    fence_mbar_init();
  }

  // ---------------- Q: scale, quantize, block mean
  float x[4][8];
  float lmax = 0.f;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int r = rg + 16 * kk;
    if (r < n) {
      load8(p.q + (row0 + r) * kHeadDim + 8 * chunk, x[kk]);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[kk][e] = __fmul_rn(x[kk][e], p.c_s);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[kk][e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      xs[r * kHeadDim + 8 * chunk + e] = x[kk][e];
      lmax = fmaxf(lmax, fabsf(x[kk][e]));
    }
  }
  float s = __fdiv_rn(block_max(lmax, red), 127.f);
  store_codes(x, s, p.q8 + prow0 * kHeadDim, rg, chunk);
  if (tid == 0) p.q_scale[blk] = s;
  if (tid < kHeadDim) {
    float acc = 0.f;
    for (int r = 0; r < n; ++r) acc = __fadd_rn(acc, xs[r * kHeadDim + tid]);
    p.q_bar[blk * kHeadDim + tid] = __fdiv_rn(acc, static_cast<float>(n));
  }
  __syncthreads();

  // ---------------- K: smooth, quantize, block mean, phi(K~) for the linear state
  lmax = 0.f;
  float mu8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mu8[e] = p.mu[bh * kHeadDim + 8 * chunk + e];
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int r = rg + 16 * kk;
    if (r < n) {
      load8(p.k + (row0 + r) * kHeadDim + 8 * chunk, x[kk]);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[kk][e] = __fsub_rn(x[kk][e], mu8[e]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[kk][e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      xs[r * kHeadDim + 8 * chunk + e] = x[kk][e];
      lmax = fmaxf(lmax, fabsf(x[kk][e]));
    }
  }
  s = __fdiv_rn(block_max(lmax, red), 127.f);
  store_codes(x, s, p.k8 + prow0 * kHeadDim, rg, chunk);
  if (tid == 0) p.k_scale[blk] = s;

  // V rows -> MN-major SW128 tile (zeros for padded tokens)
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int r = rg + 16 * kk;
    uint4 u = make_uint4(0, 0, 0, 0);
    if (r < n) u = *reinterpret_cast<const uint4*>(p.v + (row0 + r) * kHeadDim + 8 * chunk);
    st_shared_v4(smem_u32(sB) + (chunk >> 3) * 8192 + sw128_offset(r, chunk & 7), u.x, u.y, u.z,
                 u.w);
  }

  float zacc = 0.f;
  if (tid < kHeadDim) {
    const int c = tid;
    float acc = 0.f;
    for (int r = 0; r < n; ++r) acc = __fadd_rn(acc, xs[r * kHeadDim + c]);
    p.k_bar[blk * kHeadDim + c] = __fdiv_rn(acc, static_cast<float>(n));
    // row c of phi(K~)^T: 64 tokens, bf16, padded tokens 0
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r0 = 8 * q + 2 * e;
        const float f0 = r0 < n ? phi_f32(xs[r0 * kHeadDim + c]) : 0.f;
        const float f1 = r0 + 1 < n ? phi_f32(xs[(r0 + 1) * kHeadDim + c]) : 0.f;
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
    mma_commit(smem_u32(bar));
  }
  const bool ok = mbar_wait(smem_u32(bar), 0, &abort_flag, p.status);
  tc_fence_after();

  // h_j[c][e]: TMEM lane c, column e. Warps w and w+4 split the 128 columns.
  if (ok) {
    const int c = 32 * (warp & 3) + lane;
    const int col0 = 64 * (warp >> 2);
    uint32_t rr[64];
    tmem_ld64_sync(taddr + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + col0, rr);
    uint4* dst = reinterpret_cast<uint4*>(p.h + (blk * kHeadDim + c) * kHeadDim + col0);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      dst[q] = make_uint4(pack_bf16x2(__uint_as_float(rr[8 * q]), __uint_as_float(rr[8 * q + 1])),
                          pack_bf16x2(__uint_as_float(rr[8 * q + 2]), __uint_as_float(rr[8 * q + 3])),
                          pack_bf16x2(__uint_as_float(rr[8 * q + 4]), __uint_as_float(rr[8 * q + 5])),
                          pack_bf16x2(__uint_as_float(rr[8 * q + 6]), __uint_as_float(rr[8 * q + 7])));
#pragma unroll
    for (int q = 0; q < 4; ++q)
      dst[4 + q] =
          make_uint4(pack_bf16x2(__uint_as_float(rr[32 + 8 * q]), __uint_as_float(rr[32 + 8 * q + 1])),
                     pack_bf16x2(__uint_as_float(rr[32 + 8 * q + 2]), __uint_as_float(rr[32 + 8 * q + 3])),
                     pack_bf16x2(__uint_as_float(rr[32 + 8 * q + 4]), __uint_as_float(rr[32 + 8 * q + 5])),
                     pack_bf16x2(__uint_as_float(rr[32 + 8 * q + 6]), __uint_as_float(rr[32 + 8 * q + 7])));
  }
  if (tid < kHeadDim) p.z[blk * kHeadDim + tid] = zacc;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(taddr, 128);
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
    prep_block_kernel<<<dim3(g.nB, g.BH), kPrepThreads, kPrepSmem, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace sgs
