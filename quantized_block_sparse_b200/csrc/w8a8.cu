// w8a8.cu - W8A8 block-wise INT8 linear layer: Y = X W^T + bias with both operands
// quantized to INT8 per 128x128 tile.
//
// Method: "TurboDiffusion Demystified", section "Pillar Three: W8A8 Linear Layer
// Quantization" (weights and activations of the linear layers in INT8, block-wise at
// 128x128 granularity) and "TurboDiffusion: Genombrottet for realtids AI-videogenerering",
// section "W8A8 Quantization". Per tile: s = fl32(amax/127), x8 = rint(fl32(x/s)) with
// ties to even; Y[m,n] = sum over 128-wide input-channel tiles kb of
// s_x[m/128,kb] * s_w[n/128,kb] * (exact integer dot of the codes), plus the bias.
//
// Kernels:
//   w8a8_quant_kernel  bf16 [R, K] -> int8 codes [R, K] and fp32 scales [ceil(R/128),
//                      ceil(K/128)]; serves activations and weights alike.
//   w8a8_gemm_kernel   persistent, one CTA per SM, 128x128 output tiles walked with the
//                      column index fastest, 128-wide K tiles (one scale per operand tile).
//                      Warp 0: TMA ring of the A/B K tiles (4 stages, K-major, 128-byte
//                      swizzle). Warp 1: tcgen05 kind::i8 MMAs (M128 N128 K32, four per K
//                      tile) into one of two 128-column TMEM partial buffers. Warps 2-9:
//                      take each K tile's partial sum out of TMEM, scale it into fp32
//                      register accumulators (packed f32x2 FMAs), add the bias and store
//                      bf16 Y.
//
// Exact int -> float without a conversion instruction: each partial buffer is preloaded
// with the bits of 1.5*2^23 and the MMAs accumulate onto it (|dot| <= 128*127^2 < 2^22),
// so the s32 result read as fp32 is 1.5*2^23 + dot exactly; one packed subtract and one
// packed FMA per two elements then add s*dot to the accumulator.
#include "../../include/sagesla.h"
#include "sagesla_internal.h"
#include "sm100_primitives.cuh"

namespace sgs {
namespace w8 {

constexpr int kTile = 128;
constexpr int kStages = 4;
constexpr int kParts = 4;  // TMEM partial buffers (128 columns each): the MMA runs up to 3 K tiles ahead
constexpr int kStageBytes = 2 * kTile * kTile;  // A and B K tiles, int8, K-major SW128
constexpr int kThreads = 320;
constexpr int kMaxKT = 128;                     // K <= 16384
constexpr int kSmem = kStages * kStageBytes + 1024 + 256 + 8 * kMaxKT * 4;
constexpr uint32_t kMagicBits = 0x4B400000u;    // 1.5 * 2^23

__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// Store one value into 32 consecutive TMEM columns of this thread's lane (the same register
// for every operand).
__device__ __forceinline__ void tmem_st32_fill(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
      "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr), "r"(v)
      : "memory");
}

// ------------------------------------------------------------------ activations -> INT8
// One CTA per 128x128 tile, 256 threads: thread t covers row t/2, columns 64*(t%2)..+63.
__global__ void __launch_bounds__(256) w8a8_quant_kernel(const __nv_bfloat16* __restrict__ x,
                                                         int8_t* __restrict__ x8,
                                                         float* __restrict__ sx, int M, int K) {
  __shared__ float wmax[8];
  const int kb = blockIdx.x, mb = blockIdx.y, t = threadIdx.x;
  const int r = mb * kTile + (t >> 1), c0 = kb * kTile + 64 * (t & 1);
  float v[64];
  float a = 0.f;
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const int c = c0 + 8 * g;
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (r < M && c < K) u = *reinterpret_cast<const uint4*>(x + static_cast<size_t>(r) * K + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * g + 2 * e] = __uint_as_float(w[e] << 16);
      v[8 * g + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
#pragma unroll
  for (int e = 0; e < 64; ++e) a = fmaxf(a, fabsf(v[e]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((t & 31) == 0) wmax[t >> 5] = a;
  __syncthreads();
  a = wmax[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) a = fmaxf(a, wmax[w]);
  const float s = __fdiv_rn(a, 127.f);
  if (t == 0) sx[static_cast<size_t>(mb) * gridDim.x + kb] = s;
  if (r >= M) return;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int c = c0 + 16 * g;
    uint32_t pk[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float y = s > 0.f ? rintf(__fdiv_rn(v[16 * g + 4 * e + b], s)) : 0.f;
        const int q = max(-127, min(127, static_cast<int>(y)));
        word |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * b);
      }
      pk[e] = word;
    }
    if (c + 16 <= K) {
      *reinterpret_cast<uint4*>(x8 + static_cast<size_t>(r) * K + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    } else {
      for (int e = 0; e < 16 && c + e < K; ++e)
        x8[static_cast<size_t>(r) * K + c + e] = static_cast<int8_t>((pk[e >> 2] >> (8 * (e & 3))) & 0xFFu);
    }
  }
}

// ------------------------------------------------------------------ the GEMM
__global__ void __launch_bounds__(kThreads, 1) w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tmX,
                                                                const __grid_constant__ CUtensorMap tmW,
                                                                const float* __restrict__ sx,
                                                                const float* __restrict__ sw,
                                                                const float* __restrict__ bias,
                                                                __nv_bfloat16* __restrict__ y,
                                                                int M, int N, int K, int n_nt,
                                                                int n_tiles, int* status) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* pfull = bars + 2 * kStages;  // [kParts] partial sum of a K tile ready (MMA commit)
  uint64_t* pfree = pfull + kParts;      // [kParts] partial read and re-armed (256 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pfree + kParts);
  float* sscale = reinterpret_cast<float*>(smem + kStages * kStageBytes + 256);  // [8][kMaxKT]
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nKT = (K + kTile - 1) / kTile;

  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    for (int b = 0; b < kParts; ++b) {
      mbar_init(smem_u32(pfull + b), 1);
      mbar_init(smem_u32(pfree + b), 256);
    }
    fence_mbar_init();
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 128 * kParts);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const int nt = tile % n_nt, mt = tile / n_nt;
        for (int kb = 0; kb < nKT; ++kb, ++it) {
          const int s = it % kStages;
          if (it >= kStages &&
              !mbar_wait(smem_u32(empty + s), ((it / kStages) - 1) & 1, &abort_flag, status)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + s * kStageBytes);
          mbar_expect_tx(smem_u32(full + s), kStageBytes);
          tma_load_3d(sa, &tmX, smem_u32(full + s), kb * kTile, mt * kTile, 0);
          tma_load_3d(sa + kTile * kTile, &tmW, smem_u32(full + s), kb * kTile, nt * kTile, 0);
        }
      }
      for (int u = max(0, it - kStages); u < it; ++u)
        mbar_wait_inflight(smem_u32(full + (u % kStages)), (u / kStages) & 1, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(2, 1, 0, 0, 128, 128);  // s32 += s8 . s8
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < nKT; ++kb, ++it) {
          const int s = it % kStages, b = it % kParts;
          if (!mbar_wait(smem_u32(pfree + b), (it / kParts) & 1, &abort_flag, status) ||
              !mbar_wait(smem_u32(full + s), (it / kStages) & 1, &abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * kStageBytes);
          const uint32_t sb = sa + kTile * kTile;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // K = 32 bytes per MMA; onto the preloaded magic
            mma_i8(taddr + 128 * b, make_sdesc(sa + 32 * kk, 16, 1024), make_sdesc(sb + 32 * kk, 16, 1024),
                   idesc, 1u);
          mma_commit(smem_u32(empty + s));
          mma_commit(smem_u32(pfull + b));
        }
      }
      if (it > 0)
        mbar_wait_inflight(smem_u32(empty + ((it - 1) % kStages)), ((it - 1) / kStages) & 1, status);
    }
  } else {
    // warps 2-9: TMEM lane quadrant warp%4, column half (warp-2)/4
    const int e = warp - 2, q = warp & 3, h = e >> 2;
    const uint32_t lane_base = taddr + (static_cast<uint32_t>(32 * q) << 16) + 64 * h;
    float* my_scale = sscale + e * kMaxKT;
#pragma unroll
    for (int b = 0; b < kParts; ++b) {
      tmem_st32_fill(lane_base + 128 * b, kMagicBits);
      tmem_st32_fill(lane_base + 128 * b + 32, kMagicBits);
    }
    tmem_wait_st();
    tc_fence_before();
#pragma unroll
    for (int b = 0; b < kParts; ++b) mbar_arrive(smem_u32(pfree + b));
    const uint64_t neg_magic = f2pack(-12582912.f, -12582912.f);  // -(1.5 * 2^23)
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      const int nt = tile % n_nt, mt = tile / n_nt;
      for (int kb = lane; kb < nKT; kb += 32)
        my_scale[kb] = __fmul_rn(sx[static_cast<size_t>(mt) * nKT + kb],
                                 sw[static_cast<size_t>(nt) * nKT + kb]);
      __syncwarp();
      uint64_t acc[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] = 0ull;
      for (int kb = 0; kb < nKT; ++kb, ++it) {
        const int b = it % kParts;
        ok = mbar_wait(smem_u32(pfull + b), (it / kParts) & 1, &abort_flag, status);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float s = my_scale[kb];
        const uint64_t s2 = f2pack(s, s);
        // This thread's 64 columns in two halves; the buffer is re-armed and released after
        // the second load, before that half's arithmetic, so the MMAs of the next K tiles
        // (up to kParts - 1 ahead) overlap the scaling.
        uint32_t r[32];
        tmem_ld32_sync(lane_base + 128 * b, r);  // columns 0-31 of this thread's half
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint64_t xv = add2(f2pack(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), neg_magic);
          acc[c] = fma2(s2, xv, acc[c]);
        }
        tmem_ld32_sync(lane_base + 128 * b + 32, r);  // columns 32-63
        tmem_st32_fill(lane_base + 128 * b, kMagicBits);  // re-arm for K tile it + kParts
        tmem_st32_fill(lane_base + 128 * b + 32, kMagicBits);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(pfree + b));
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint64_t xv = add2(f2pack(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), neg_magic);
          acc[16 + c] = fma2(s2, xv, acc[16 + c]);
        }
      }
      if (!ok) break;
      const int row = mt * kTile + 32 * q + lane;
      const int col0 = nt * kTile + 64 * h;
      if (row < M) {
        __nv_bfloat16* dst = y + static_cast<size_t>(row) * N + col0;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          float f[8];
#pragma unroll
          for (int u = 0; u < 4; ++u) f2unpack(acc[4 * g + u], f[2 * u], f[2 * u + 1]);
          const int c = col0 + 8 * g;
          if (bias) {
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] += (c + u < N) ? bias[c + u] : 0.f;
          }
          if (c + 8 <= N) {
            *reinterpret_cast<uint4*>(dst + 8 * g) =
                make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                           pack_bf16x2(f[6], f[7]));
          } else {
            for (int u = 0; u < 8 && c + u < N; ++u) dst[8 * g + u] = __float2bfloat16_rn(f[u]);
          }
        }
      }
      __syncwarp();  // my_scale is rewritten by the next tile
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(taddr, 128 * kParts);
}

}  // namespace w8
}  // namespace sgs

// ------------------------------------------------------------------ host
namespace {
bool al16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

extern "C" int sagesla_w8a8_quantize(const void* x, int rows, int K, int8_t* x8, float* scale,
                                     void* stream) {
  if (rows < 1 || K < 16 || (K % 16) != 0) return SAGESLA_ERR_INVALID_ARG;
  if (!al16(x) || !al16(x8) || !scale) return SAGESLA_ERR_INVALID_ARG;
  const long long n_rt = (static_cast<long long>(rows) + sgs::w8::kTile - 1) / sgs::w8::kTile;
  if (n_rt > 65535) return SAGESLA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid((K + sgs::w8::kTile - 1) / sgs::w8::kTile, static_cast<unsigned>(n_rt));
  {
    sgs::TraceScope ts_("w8a8_quant_kernel", st);
    sgs::w8::w8a8_quant_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), x8,
                                                     scale, rows, K);
  }
  return cudaGetLastError() == cudaSuccess ? SAGESLA_OK : SAGESLA_ERR_CUDA;
}

extern "C" int sagesla_w8a8_linear(const int8_t* x8, const float* sx, const int8_t* w8,
                                   const float* sw, const float* bias, void* y, int M, int N,
                                   int K, void* workspace, size_t workspace_bytes, void* stream) {
  if (M < 1 || N < 8 || K < 16 || (K % 16) != 0 || (N % 8) != 0) return SAGESLA_ERR_INVALID_ARG;
  if (K > sgs::w8::kTile * sgs::w8::kMaxKT) return SAGESLA_ERR_UNSUPPORTED;
  if (!al16(x8) || !al16(w8) || !al16(y) || !sx || !sw || !al16(workspace) || workspace_bytes < 256)
    return SAGESLA_ERR_INVALID_ARG;
  CUtensorMap tmX, tmW;
  if (!sgs::make_tmap_3d(&tmX, x8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, 1, 128, 128) ||
      !sgs::make_tmap_3d(&tmW, w8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, 1, 128, 128))
    return SAGESLA_ERR_CUDA;
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return SAGESLA_ERR_CUDA;
  const long long n_nt = (N + sgs::w8::kTile - 1) / sgs::w8::kTile;
  const long long n_mt = (static_cast<long long>(M) + sgs::w8::kTile - 1) / sgs::w8::kTile;
  const long long n_tiles = n_nt * n_mt;
  if (n_tiles > 0x7fffffffLL) return SAGESLA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(sgs::w8::w8a8_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           sgs::w8::kSmem) != cudaSuccess)
    return SAGESLA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    sgs::TraceScope ts_("w8a8_gemm_kernel", st);
    sgs::w8::w8a8_gemm_kernel<<<static_cast<int>(n_tiles < n_sm ? n_tiles : n_sm), sgs::w8::kThreads,
                                sgs::w8::kSmem, st>>>(
        tmX, tmW, sx, sw, bias, static_cast<__nv_bfloat16*>(y), M, N, K, static_cast<int>(n_nt),
        static_cast<int>(n_tiles), static_cast<int*>(workspace));
  }
  return cudaGetLastError() == cudaSuccess ? SAGESLA_OK : SAGESLA_ERR_CUDA;
}
