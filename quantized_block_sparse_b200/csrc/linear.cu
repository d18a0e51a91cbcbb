// linear.cu - the linear-attention branch for marginal key blocks.
//
// Method: "TurboDiffusion Demystified", section "Pillar Two: Sparse-Linear Attention -
// SLA": the key blocks that are neither kept exactly nor skipped are covered by a light
// linear-attention term. With phi(x) = elu(x) + 1 and the per-key-block states
// h_j = phi(K~_j)^T V_j, z_j = phi(K~_j)^T 1 written by prepare:
//   H_i = sum_{j marginal for i} h_j,  Z_i = sum_{j marginal} z_j,
//   O_l[t] = phi(Q~_t)^T H_i / (phi(Q~_t) . Z_i).
//
// Kernels:
//   hgemm_kernel   H = M . h per head, M the 0/1 marginal mask [nB x nBp] and h viewed as
//                  [nB x d*d]: a persistent tcgen05 bf16 GEMM (fp32 accumulation in two
//                  TMEM accumulators), 128x256 output tiles, TMA-fed 4-stage pipeline,
//                  bf16 output; plus one 256-column tile for Z.
//   zb_kernel      z_j split into two bf16 parts, z_hi = bf16(z) and z_lo = bf16(z - z_hi);
//                  hgemm_kernel's extra column tile multiplies M by [z_hi | z_lo] (exact
//                  0/1 x bf16 products, fp32 accumulation) and Z = M.z_hi + M.z_lo in fp32,
//                  so Z keeps about 17 significant bits of z instead of bf16's 8.
// phi(Q~) H_i / phi(Q~) . Z_i itself is formed in the attention kernel's epilogue (the
// H_i tiles stream through its V ring; the product lands in TMEM next to O_s).
#include "sagesla_internal.h"
#include "sm100_primitives.cuh"

namespace sgs {
namespace {

// ------------------------------------------------------------------ H = M . h
// Persistent tcgen05 GEMM, one CTA per SM: each CTA walks output tiles (128 query blocks x
// 256 columns of h's d*d, N fastest so consecutive tiles share the mask tile in L2; 256-wide
// tiles halve the mask re-reads, the main L2 traffic). Warp 0 streams A/B k-blocks through
// a 4-stage ring with TMA, warp 1 issues the MMAs (M128 N256 K16) into one of two 256-column
// TMEM accumulators, warps 2-5 drain the other accumulator (bf16) while the next tile runs.
// One more 256-column tile per row block computes M . [z_hi | z_lo] (z split into two bf16
// parts by zb_kernel); its drain adds the two halves and writes Z in fp32.
constexpr int kGemmStages = 4;
constexpr int kGemmStageBytes = 16384 + 32768;
constexpr int kGemmThreads = 192;
constexpr int kGemmSmem = kGemmStages * kGemmStageBytes + 1024 + 256;

__global__ void __launch_bounds__(kGemmThreads, 1) hgemm_kernel(const __grid_constant__ CUtensorMap tmA,
                                                             const __grid_constant__ CUtensorMap tmB,
                                                             const __grid_constant__ CUtensorMap tmZ,
                                                             __nv_bfloat16* __restrict__ Hout,
                                                             float* __restrict__ Zout, int nB,
                                                             int n_mt, int n_tiles, int* status) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemmStages * kGemmStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kGemmStages;
  uint64_t* tfull = bars + 2 * kGemmStages;   // [2] accumulator ready
  uint64_t* tempty = tfull + 2;               // [2] accumulator drained
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  __shared__ int abort_flag;

  constexpr int kNTH = kHeadDim * kHeadDim / 256;  // 64 N-tiles of H
  constexpr int kNT = kNTH + 1;                     // + the Z tile
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nK = (nB + 63) / 64;

  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(tfull + a), 1);
      mbar_init(smem_u32(tempty + a), 128);
    }
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmZ);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;  // k-block counter across tiles (ring position)
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const int nt = tile % kNT, mt = (tile / kNT) % n_mt, bh = tile / (kNT * n_mt);
        for (int kb = 0; kb < nK; ++kb, ++it) {
          const int s = it % kGemmStages;
          if (it >= kGemmStages &&
              !mbar_wait(smem_u32(empty + s), ((it / kGemmStages) - 1) & 1, &abort_flag, status)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + s * kGemmStageBytes);
          const uint32_t sb = sa + 16384;
          mbar_expect_tx(smem_u32(full + s), kGemmStageBytes);
          tma_load_3d(sa, &tmA, smem_u32(full + s), kb * 64, mt * 128, bh);
          if (nt < kNTH) {
#pragma unroll
            for (int g = 0; g < 4; ++g)
              tma_load_3d(sb + 8192 * g, &tmB, smem_u32(full + s), nt * 256 + 64 * g, kb * 64, bh);
          } else {
#pragma unroll
            for (int g = 0; g < 4; ++g)
              tma_load_3d(sb + 8192 * g, &tmZ, smem_u32(full + s), 64 * g, kb * 64, bh);
          }
        }
      }
      // copies still in flight land before the CTA exits
      for (int u = max(0, it - kGemmStages); u < it; ++u)
        mbar_wait_inflight(smem_u32(full + (u % kGemmStages)), (u / kGemmStages) & 1, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(1, 1, 0, 1, 128, 256);
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++lt) {
        const int a = lt & 1;
        if (lt >= 2 && !mbar_wait(smem_u32(tempty + a), ((lt >> 1) - 1) & 1, &abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < nK; ++kb, ++it) {
          const int s = it % kGemmStages;
          if (!mbar_wait(smem_u32(full + s), (it / kGemmStages) & 1, &abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * kGemmStageBytes);
          const uint32_t sb = sa + 16384;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(taddr + 256 * a, make_sdesc(sa + kk * 32, 16, 1024),
                     make_sdesc(sb + kk * 2048, 8192, 1024), idesc, (kb | kk) != 0);
          mma_commit(smem_u32(empty + s));
        }
        if (ok) mma_commit(smem_u32(tfull + a));
      }
      // every MMA issued completes before the CTA releases TMEM (the last empty commit)
      if (it > 0) mbar_wait_inflight(smem_u32(empty + ((it - 1) % kGemmStages)), ((it - 1) / kGemmStages) & 1, status);
    }
  } else {
    // epilogue warps 2-5: TMEM lane quadrant w%4 -> rows 32*(w%4) .. of the tile
    const int wq = warp & 3;
    int lt = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++lt) {
      const int a = lt & 1;
      const int nt = tile % kNT, mt = (tile / kNT) % n_mt, bh = tile / (kNT * n_mt);
      const bool ok = mbar_wait(smem_u32(tfull + a), (lt >> 1) & 1, &abort_flag, status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int i = mt * 128 + 32 * wq + lane;
      if (nt < kNTH) {
        __nv_bfloat16* dst = Hout + (static_cast<size_t>(bh) * nB + i) * (kHeadDim * kHeadDim) + nt * 256;
#pragma unroll
        for (int cchunk = 0; cchunk < 8; ++cchunk) {
          uint32_t r[32];
          tmem_ld32_sync(taddr + (static_cast<uint32_t>(32 * wq) << 16) + 256 * a + 32 * cchunk, r);
          if (i < nB) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * cchunk);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              d4[q] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * q]), __uint_as_float(r[8 * q + 1])),
                                 pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3])),
                                 pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5])),
                                 pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7])));
          }
        }
      } else {
        // columns [0,128): M . z_hi, [128,256): M . z_lo; Z = their fp32 sum
        float* dst = Zout + (static_cast<size_t>(bh) * nB + i) * kHeadDim;
#pragma unroll
        for (int cchunk = 0; cchunk < 4; ++cchunk) {
          uint32_t rh[32], rl[32];
          const uint32_t ta = taddr + (static_cast<uint32_t>(32 * wq) << 16) + 256 * a + 32 * cchunk;
          tmem_ld32_sync(ta, rh);
          tmem_ld32_sync(ta + 128, rl);
          if (i < nB) {
            float4* d4 = reinterpret_cast<float4*>(dst + 32 * cchunk);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float f[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                f[e] = __fadd_rn(__uint_as_float(rh[4 * q + e]), __uint_as_float(rl[4 * q + e]));
              d4[q] = make_float4(f[0], f[1], f[2], f[3]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(tempty + a));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(taddr, 512);
}

// ------------------------------------------------------------------ z -> bf16 hi + lo
// The B operand of the Z column tile of hgemm_kernel: row j of zb is [z_hi | z_lo] (2 x 128
// bf16), z_hi = bf16(z_j) and z_lo = bf16(z_j - z_hi) (the subtraction is exact), both RNE.
// x indexes groups of 4 channels: row j = x / 32, channels 4*(x % 32) .. +3.
__device__ __forceinline__ float bf16_round(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}
__global__ void __launch_bounds__(256) zb_kernel(const float4* __restrict__ z,
                                                 uint2* __restrict__ zb, size_t n4) {
  for (size_t x = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; x < n4;
       x += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = z[x];
    const float4 h = make_float4(bf16_round(v.x), bf16_round(v.y), bf16_round(v.z), bf16_round(v.w));
    const size_t row = x >> 5, c4 = x & 31;
    zb[row * 64 + c4] = make_uint2(pack_bf16x2(h.x, h.y), pack_bf16x2(h.z, h.w));
    zb[row * 64 + 32 + c4] = make_uint2(pack_bf16x2(v.x - h.x, v.y - h.y), pack_bf16x2(v.z - h.z, v.w - h.w));
  }
}

}  // namespace

// Sums of per-key-block states over a 0/1 block mask, per head: Hout[i] = sum_j M[i][j] h[j]
// (bf16 [nB, d*d]) and Zout[i] = sum_j M[i][j] z[j] (fp32 [nB, d]); M bf16 [nB, nBp].
// zb is scratch for the hi/lo split of z (bf16 [BH, nB, 2d]).
cudaError_t launch_mask_gemm(const Dims& g, const void* mask, const void* h, const float* z,
                             __nv_bfloat16* Hout, float* Zout, __nv_bfloat16* zb, int* status,
                             cudaStream_t st) {
  CUtensorMap tmA, tmB, tmZ;
  if (!make_tmap_3d(&tmA, mask, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.nBp, g.nB, g.BH, 64, 128) ||
      !make_tmap_3d(&tmB, h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kHeadDim * kHeadDim, g.nB, g.BH, 64,
                    64) ||
      !make_tmap_3d(&tmZ, zb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 2 * kHeadDim, g.nB, g.BH, 64, 64))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(hgemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e != cudaSuccess) return e;
  {
    TraceScope ts_("zb_kernel", st);
    const size_t n4 = static_cast<size_t>(g.BH) * g.nB * kHeadDim / 4;
    const int blocks = static_cast<int>((n4 + 255) / 256 < 4096 ? (n4 + 255) / 256 : 4096);
    zb_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const float4*>(z), reinterpret_cast<uint2*>(zb), n4);
  }
  {
    TraceScope ts_("hgemm_kernel", st);
    const int n_mt = (g.nB + 127) / 128;
    const int n_tiles = (kHeadDim * kHeadDim / 256 + 1) * n_mt * g.BH;
    int dev = 0, n_sm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    const int grid = n_tiles < n_sm ? n_tiles : n_sm;
    hgemm_kernel<<<grid, kGemmThreads, kGemmSmem, st>>>(tmA, tmB, tmZ, Hout, Zout, g.nB, n_mt, n_tiles,
                                                         status);
  }
  return cudaGetLastError();
}

cudaError_t launch_linear(const Dims& g, const void* mask, int m, const void* h, const float* z,
                          char* ws, cudaStream_t st) {
  if (m == 0) return cudaSuccess;
  const WsLayout L = ws_layout(g);
  return launch_mask_gemm(g, mask, h, z, reinterpret_cast<__nv_bfloat16*>(ws + L.Hbuf),
                          reinterpret_cast<float*>(ws + L.Zbuf), reinterpret_cast<__nv_bfloat16*>(ws + L.Zb),
                          reinterpret_cast<int*>(ws + L.status), st);
}

}  // namespace sgs
