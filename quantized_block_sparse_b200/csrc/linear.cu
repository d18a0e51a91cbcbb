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
//   linout_kernel  per pair of adjacent query blocks: phi(Q~) (recomputed from Q, bf16)
//                  times H_i on tcgen05 (M = 128 rows = both blocks, one MMA chain per
//                  block), divided by phi(Q~) . Z_i; bf16 O_l for the attention epilogue.
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

// ------------------------------------------------------------------ O_l
// One CTA per pair of query blocks, 256 threads. Every load is issued at the start by TMA:
// H_i0 and H_i1 (64 KB), and the pair's Q rows straight into the 128-byte-swizzled
// K-major A tile, where phi(Q~) is computed in place (thread t: row t%128, channels
// [64*(t/128), +64)) together with its part of the denominator. Eight warps then read the
// two 128x128 products back (a quadrant of rows and half of the columns each), scale by
// 1/den and stage O_l over the H tiles (swizzled) for four TMA stores.
constexpr int kLinThreads = 256;
constexpr int kLinSmem = 32768 + 65536 + 1024 + 1024 + 1024 + 256;

__global__ void __launch_bounds__(kLinThreads) linout_kernel(const __grid_constant__ CUtensorMap tmH,
                                                             const __grid_constant__ CUtensorMap tmQ,
                                                             const __grid_constant__ CUtensorMap tmO,
                                                             const float* __restrict__ Z, float c_s,
                                                             int N, int nB, int* status) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sA = smem;            // Q, then phi(Q~): 2 column blocks x 128 rows x 128 B
  unsigned char* sH = smem + 32768;    // H_i0, H_i1: each 2 e-groups x 128 c rows x 128 B
  float* dpart = reinterpret_cast<float*>(smem + 32768 + 65536);         // [2][128] denominator halves
  float* sZ = reinterpret_cast<float*>(smem + 32768 + 65536 + 1024);     // Z_i0, Z_i1 [2][128]
  uint64_t* lfull = reinterpret_cast<uint64_t*>(smem + 32768 + 65536 + 2048);  // Q, H, Z landed
  uint64_t* mdone = lfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);
  __shared__ int abort_flag;

  const int pr = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = 2 * pr;
  const bool two = (i0 + 1) < nB;
  if (tid == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(lfull), 1);
    mbar_init(smem_u32(mdone), 1);
    fence_mbar_init();
    mbar_expect_tx(smem_u32(lfull), (two ? 65536 + 1024 : 32768 + 512) + 32768);
    for (int b = 0; b < (two ? 2 : 1); ++b)
      bulk_load(smem_u32(sZ) + b * 512, Z + (static_cast<size_t>(bh) * nB + i0 + b) * kHeadDim, 512,
                smem_u32(lfull));
    for (int b = 0; b < (two ? 2 : 1); ++b) {
      const uint32_t dst = smem_u32(sH) + b * 32768;
      tma_load_3d(dst, &tmH, smem_u32(lfull), 0, (i0 + b) * 128, bh);
      tma_load_3d(dst + 16384, &tmH, smem_u32(lfull), 64, (i0 + b) * 128, bh);
    }
    // Q rows of blocks i0 and i0+1 (rows past N read as zero), channel halves 0-63 / 64-127
    for (int cb = 0; cb < 2; ++cb)
      for (int b = 0; b < 2; ++b)
        tma_load_3d(smem_u32(sA) + cb * 16384 + b * 8192, &tmQ, smem_u32(lfull), 64 * cb, (i0 + b) * 64, bh);
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;
  bool ok = mbar_wait(smem_u32(lfull), 0, &abort_flag, status);
  if (!ok) mbar_wait_inflight(smem_u32(lfull), 0, status);

  // phi(Q~) in place for (row r, 64 channels) and that part of phi(Q~).Z_i, with the
  // bf16-rounded phi values the tensor core sees. phi is rounded to bf16, so the fast
  // exponential (relative error ~2^-21) is enough.
  {
    const int r = tid & 127, chh = tid >> 7;
    const int i = i0 + (r >> 6);
    const float* zr = sZ + ((i < nB) ? (r >> 6) : 0) * kHeadDim + 64 * chh;
    const uint32_t tile = smem_u32(sA) + chh * 16384;
    float dacc = 0.f;
#pragma unroll
    for (int cb = 0; cb < 8; ++cb) {  // 8 channels per 16-byte chunk
      const uint32_t addr = tile + sw128_offset(r, cb);
      uint32_t w[4];
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr));
      const float4 z0 = *reinterpret_cast<const float4*>(zr + 8 * cb);
      const float4 z1 = *reinterpret_cast<const float4*>(zr + 8 * cb + 4);
      const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w[e]));
        const float x0 = __fmul_rn(f.x, c_s), x1 = __fmul_rn(f.y, c_s);
        const float p0 = x0 > 0.f ? x0 + 1.f : __expf(x0);
        const float p1 = x1 > 0.f ? x1 + 1.f : __expf(x1);
        w[e] = pack_bf16x2(p0, p1);
        const float2 pr2 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w[e]));
        dacc = fmaf(pr2.x, zz[2 * e], dacc);
        dacc = fmaf(pr2.y, zz[2 * e + 1], dacc);
      }
      st_shared_v4(addr, w[0], w[1], w[2], w[3]);
    }
    dpart[chh * 128 + r] = dacc;
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (tid == 0) {
    if (ok) {
      constexpr uint32_t idesc = make_idesc(1, 1, 0, 1, 128, 128);
      for (int b = 0; b < (two ? 2 : 1); ++b) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = make_sdesc(smem_u32(sA) + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = make_sdesc(smem_u32(sH) + b * 32768 + kk * 2048, 16384, 1024);
          mma_bf16(taddr + 128 * b, a, bd, idesc, kk > 0);
        }
      }
    }
    mma_commit(smem_u32(mdone));
  }
  __syncwarp();
  ok = mbar_wait(smem_u32(mdone), 0, &abort_flag, status) && ok;
  tc_fence_after();
  // Warp w: TMEM lane quadrant w%4 (rows 32*(w%4) ..), output columns [64*(w/4), +64).
  // Rows 0-63 (block i0) read the product with H_i0 (columns 0-127), rows 64-127 the one
  // with H_i0+1 (columns 128-255). O_l is staged over the H tiles (free once the MMAs
  // are done): column half ch2 at sH + 16 KB * ch2, 128 rows x 128 B, swizzled.
  const int wq = warp & 3, ch2 = warp >> 2;
  const int r = 32 * wq + lane;
  const int half = wq >> 1;
  if (ok && (i0 + half < nB)) {  // warp-uniform
    const float inv = 1.f / (dpart[r] + dpart[128 + r]);
    const uint32_t tile = smem_u32(sH) + ch2 * 16384;
#pragma unroll
    for (int cchunk = 0; cchunk < 2; ++cchunk) {
      uint32_t rr[32];
      tmem_ld32_sync(taddr + (static_cast<uint32_t>(32 * wq) << 16) + 128 * half + 64 * ch2 + 32 * cchunk, rr);
#pragma unroll
      for (int qq = 0; qq < 4; ++qq)
        st_shared_v4(tile + sw128_offset(r, 4 * cchunk + qq),
                     pack_bf16x2(__uint_as_float(rr[8 * qq]) * inv, __uint_as_float(rr[8 * qq + 1]) * inv),
                     pack_bf16x2(__uint_as_float(rr[8 * qq + 2]) * inv, __uint_as_float(rr[8 * qq + 3]) * inv),
                     pack_bf16x2(__uint_as_float(rr[8 * qq + 4]) * inv, __uint_as_float(rr[8 * qq + 5]) * inv),
                     pack_bf16x2(__uint_as_float(rr[8 * qq + 6]) * inv, __uint_as_float(rr[8 * qq + 7]) * inv));
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(taddr, 256);
  if (tid == 0 && ok) {  // rows past N fall outside the tensor and are not written
    for (int b = 0; b < (two ? 2 : 1); ++b)
      for (int cb = 0; cb < 2; ++cb)
        tma_store_3d(&tmO, smem_u32(sH) + cb * 16384 + b * 8192, 64 * cb, (i0 + b) * 64, bh);
    bulk_store_commit_wait_read();
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

cudaError_t launch_linear(const Dims& g, const void* q, float sm_scale, const void* mask,
                          const int32_t* marg, int m, const void* h, const float* z, char* ws,
                          cudaStream_t st) {
  if (m == 0) return cudaSuccess;
  const WsLayout L = ws_layout(g);
  int* status = reinterpret_cast<int*>(ws + L.status);
  __nv_bfloat16* Hbuf = reinterpret_cast<__nv_bfloat16*>(ws + L.Hbuf);
  float* Zbuf = reinterpret_cast<float*>(ws + L.Zbuf);
  __nv_bfloat16* Ol = reinterpret_cast<__nv_bfloat16*>(ws + L.Ol);
  __nv_bfloat16* Zb = reinterpret_cast<__nv_bfloat16*>(ws + L.Zb);

  cudaError_t e = launch_mask_gemm(g, mask, h, z, Hbuf, Zbuf, Zb, status, st);
  if (e != cudaSuccess) return e;
  CUtensorMap tmH, tmQ, tmO;
  if (!make_tmap_3d(&tmH, Hbuf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kHeadDim,
                    static_cast<uint64_t>(g.nB) * kHeadDim, g.BH, 64, 128) ||
      !make_tmap_3d(&tmQ, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kHeadDim, g.N, g.BH, 64, 64) ||
      !make_tmap_3d(&tmO, Ol, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kHeadDim, g.N, g.BH, 64, 64))
    return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(linout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kLinSmem);
  if (e != cudaSuccess) return e;
  {
    TraceScope ts_("linout_kernel", st);
    linout_kernel<<<dim3((g.nB + 1) / 2, g.BH), kLinThreads, kLinSmem, st>>>(tmH, tmQ, tmO, Zbuf, sm_scale,
                                                                          g.N, g.nB, status);
  }
  return cudaGetLastError();
}

}  // namespace sgs
