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
//                  [nB x d*d]: a tcgen05 bf16 GEMM (fp32 accumulation in TMEM), 128x128
//                  output tiles, TMA-fed 3-stage pipeline, bf16 output.
//   zsum_kernel    Z_i = sum of z_j over the marginal blocks (mask row), fp32, ascending j.
//   linout_kernel  per pair of query blocks: phi(Q~) (recomputed from Q, bf16) times H_i
//                  on tcgen05 (M = 128 rows = both blocks, one MMA chain per block),
//                  divided by phi(Q~) . Z_i; bf16 O_l for the attention epilogue.
#include "sagesla_internal.h"
#include "sm100_primitives.cuh"

namespace sgs {
namespace {

// ------------------------------------------------------------------ H = M . h
constexpr int kGemmStages = 3;
constexpr int kGemmStageBytes = 16384 + 16384;
constexpr int kGemmSmem = kGemmStages * kGemmStageBytes + 1024 + 256;

__global__ void __launch_bounds__(128) hgemm_kernel(const __grid_constant__ CUtensorMap tmA,
                                                    const __grid_constant__ CUtensorMap tmB,
                                                    __nv_bfloat16* __restrict__ Hout, int nB,
                                                    int* status) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemmStages * kGemmStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kGemmStages;
  uint64_t* done = bars + 2 * kGemmStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  __shared__ int abort_flag;

  const int nt = blockIdx.x, mt = blockIdx.y, bh = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nK = (nB + 63) / 64;

  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    mbar_init(smem_u32(done), 1);
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;

  if (warp == 0 && lane == 0) {
    for (int kb = 0; kb < nK; ++kb) {
      const int s = kb % kGemmStages;
      if (kb >= kGemmStages &&
          !mbar_wait(smem_u32(empty + s), ((kb / kGemmStages) - 1) & 1, &abort_flag, status))
        break;
      const uint32_t sa = smem_u32(smem + s * kGemmStageBytes);
      const uint32_t sb = sa + 16384;
      mbar_expect_tx(smem_u32(full + s), kGemmStageBytes);
      tma_load_3d(sa, &tmA, smem_u32(full + s), kb * 64, mt * 128, bh);
      tma_load_3d(sb, &tmB, smem_u32(full + s), nt * 128, kb * 64, bh);
      tma_load_3d(sb + 8192, &tmB, smem_u32(full + s), nt * 128 + 64, kb * 64, bh);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = make_idesc(1, 1, 0, 1, 128, 128);
    bool ok = true;
    for (int kb = 0; kb < nK && ok; ++kb) {
      const int s = kb % kGemmStages;
      ok = mbar_wait(smem_u32(full + s), (kb / kGemmStages) & 1, &abort_flag, status);
      if (!ok) break;
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * kGemmStageBytes);
      const uint32_t sb = sa + 16384;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(taddr, make_sdesc(sa + kk * 32, 16, 1024), make_sdesc(sb + kk * 2048, 8192, 1024),
                 idesc, (kb | kk) != 0);
      mma_commit(smem_u32(empty + s));
    }
    mma_commit(smem_u32(done));
  }
  __syncwarp();
  const bool ok = mbar_wait(smem_u32(done), 0, &abort_flag, status);
  tc_fence_after();
  if (ok) {
    const int i = mt * 128 + 32 * warp + lane;
    __nv_bfloat16* dst = Hout + (static_cast<size_t>(bh) * nB + i) * (kHeadDim * kHeadDim) + nt * 128;
#pragma unroll
    for (int cchunk = 0; cchunk < 4; ++cchunk) {
      uint32_t r[32];
      tmem_ld32_sync(taddr + (static_cast<uint32_t>(32 * warp) << 16) + 32 * cchunk, r);
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(taddr, 128);
}

// ------------------------------------------------------------------ Z_i
// Z_i = sum over j of mask_ij * z_j, ascending j, one fp32 FMA per term (mask_ij is 0 or 1,
// so each step adds z_j exactly once or leaves the sum unchanged). A CTA covers 16 query
// blocks; z and the mask rows are staged in shared memory 128 key blocks at a time, so each
// z row is read from L2 once per 16 query blocks instead of once per query block.
constexpr int kZRows = 16;
constexpr int kZChunk = 128;
constexpr int kZSmem = (kZChunk * kHeadDim + kZRows * kZChunk) * 4;

__global__ void __launch_bounds__(256) zsum_kernel(const float* __restrict__ z,
                                                   const __nv_bfloat16* __restrict__ mask,
                                                   float* __restrict__ Z, int nB, int nBp) {
  extern __shared__ float zsm[];
  float* zs = zsm;                          // [kZChunk][128]
  float* ms = zsm + kZChunk * kHeadDim;     // [kZRows][kZChunk]
  const int i0 = blockIdx.x * kZRows, bh = blockIdx.y, tid = threadIdx.x;
  const int g = tid >> 7, c = tid & 127;
  const int rows = min(kZRows, nB - i0);
  const float* zh = z + static_cast<size_t>(bh) * nB * kHeadDim;
  const __nv_bfloat16* mh = mask + (static_cast<size_t>(bh) * nB + i0) * nBp;
  float acc[kZRows / 2];
#pragma unroll
  for (int r = 0; r < kZRows / 2; ++r) acc[r] = 0.f;

  for (int j0 = 0; j0 < nB; j0 += kZChunk) {
    const int jn = min(kZChunk, nB - j0), jn4 = (jn + 3) & ~3;
    __syncthreads();
    const float4* src = reinterpret_cast<const float4*>(zh + static_cast<size_t>(j0) * kHeadDim);
    for (int x = tid; x < jn * (kHeadDim / 4); x += 256) cp_async16(smem_u32(zs + 4 * x), src + x);
    cp_async_commit();
    for (int x = jn * (kHeadDim / 4) + tid; x < jn4 * (kHeadDim / 4); x += 256)
      reinterpret_cast<float4*>(zs)[x] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int t = 0; t < kZRows * kZChunk / 256; ++t) {
      const int x = tid + 256 * t;
      const int r = x / kZChunk, jj = x % kZChunk;
      ms[x] = (r < rows && jj < jn) ? __bfloat162float(mh[static_cast<size_t>(r) * nBp + j0 + jj]) : 0.f;
    }
    cp_async_wait<0>();
    __syncthreads();
    const float* mrow = ms + g * (kZRows / 2) * kZChunk;
    for (int jj = 0; jj < jn4; jj += 4) {
      const float z0 = zs[(jj + 0) * kHeadDim + c], z1 = zs[(jj + 1) * kHeadDim + c];
      const float z2 = zs[(jj + 2) * kHeadDim + c], z3 = zs[(jj + 3) * kHeadDim + c];
#pragma unroll
      for (int r = 0; r < kZRows / 2; ++r) {
        const float4 mv = *reinterpret_cast<const float4*>(mrow + r * kZChunk + jj);
        acc[r] = fmaf(mv.x, z0, acc[r]);
        acc[r] = fmaf(mv.y, z1, acc[r]);
        acc[r] = fmaf(mv.z, z2, acc[r]);
        acc[r] = fmaf(mv.w, z3, acc[r]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kZRows / 2; ++r) {
    const int row = g * (kZRows / 2) + r;
    if (row < rows) Z[(static_cast<size_t>(bh) * nB + i0 + row) * kHeadDim + c] = acc[r];
  }
}

// ------------------------------------------------------------------ O_l
// One CTA per pair of query blocks, 256 threads: thread t builds phi(Q~) for row t%128 and
// channels [64*(t/128), +64) and its part of the denominator; eight warps then read the two
// 128x128 products back, each a quadrant of rows and half of the columns.
constexpr int kLinThreads = 256;
constexpr int kLinSmem = 32768 + 65536 + 1024 + 1024 + 256;

__global__ void __launch_bounds__(kLinThreads) linout_kernel(const __grid_constant__ CUtensorMap tmH,
                                                             const __nv_bfloat16* __restrict__ q,
                                                             const float* __restrict__ Z, float c_s,
                                                             __nv_bfloat16* __restrict__ Ol, int N,
                                                             int nB, int* status) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sA = smem;            // phi(Q~): 2 column blocks x 128 rows x 128 B
  unsigned char* sH = smem + 32768;    // H_i0, H_i1: each 2 e-groups x 128 c rows x 128 B
  float* dpart = reinterpret_cast<float*>(smem + 32768 + 65536);  // [2][128] denominator halves
  uint64_t* hfull = reinterpret_cast<uint64_t*>(smem + 32768 + 65536 + 1024);
  uint64_t* mdone = hfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);
  __shared__ int abort_flag;

  const int pr = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = 2 * pr;
  const bool two = (i0 + 1) < nB;
  if (tid == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(hfull), 1);
    mbar_init(smem_u32(mdone), 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;

  if (tid == 0) {
    mbar_expect_tx(smem_u32(hfull), two ? 65536 : 32768);
    for (int b = 0; b < (two ? 2 : 1); ++b) {
      const uint32_t dst = smem_u32(sH) + b * 32768;
      tma_load_3d(dst, &tmH, smem_u32(hfull), 0, (i0 + b) * 128, bh);
      tma_load_3d(dst + 16384, &tmH, smem_u32(hfull), 64, (i0 + b) * 128, bh);
    }
  }

  // phi(Q~) for (row r, 64 channels) and that part of phi(Q~).Z_i, with the bf16-rounded
  // phi values the tensor core sees. phi is rounded to bf16, so the fast exponential
  // (relative error ~2^-21) is enough.
  {
    const int r = tid & 127, chh = tid >> 7;
    const int i = i0 + (r >> 6);
    const int t = i * 64 + (r & 63);
    const bool valid = (i < nB) && (t < N);
    const __nv_bfloat16* qr = q + (static_cast<size_t>(bh) * N + (valid ? t : 0)) * kHeadDim + 64 * chh;
    const float* zr = Z + (static_cast<size_t>(bh) * nB + (i < nB ? i : 0)) * kHeadDim + 64 * chh;
    float dacc = 0.f;
#pragma unroll
    for (int cb = 0; cb < 8; ++cb) {  // 8 channels per chunk
      uint32_t w[4] = {0, 0, 0, 0};
      if (valid) {
        const uint4 u = *reinterpret_cast<const uint4*>(qr + 8 * cb);
        const float4 z0 = *reinterpret_cast<const float4*>(zr + 8 * cb);
        const float4 z1 = *reinterpret_cast<const float4*>(zr + 8 * cb + 4);
        const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(b2[e]);
          const float x0 = __fmul_rn(f.x, c_s), x1 = __fmul_rn(f.y, c_s);
          const float p0 = x0 > 0.f ? x0 + 1.f : __expf(x0);
          const float p1 = x1 > 0.f ? x1 + 1.f : __expf(x1);
          w[e] = pack_bf16x2(p0, p1);
          const float2 pr2 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w[e]));
          dacc = fmaf(pr2.x, zz[2 * e], dacc);
          dacc = fmaf(pr2.y, zz[2 * e + 1], dacc);
        }
      }
      const int cg = 8 * chh + cb;  // 16-byte chunk index over the 128 channels
      st_shared_v4(smem_u32(sA) + (cg >> 3) * 16384 + sw128_offset(r, cg & 7), w[0], w[1], w[2], w[3]);
    }
    dpart[chh * 128 + r] = dacc;
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (tid == 0) {
    bool ok = mbar_wait(smem_u32(hfull), 0, &abort_flag, status);
    tc_fence_after();
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
    } else {
      mbar_wait_inflight(smem_u32(hfull), 0, status);
    }
    mma_commit(smem_u32(mdone));
  }
  __syncwarp();
  const bool ok = mbar_wait(smem_u32(mdone), 0, &abort_flag, status);
  tc_fence_after();
  // Warp w: TMEM lane quadrant w%4 (rows 32*(w%4) ..), output columns [64*(w/4), +64).
  // Rows 0-63 (block i0) read the product with H_i0 (columns 0-127), rows 64-127 the one
  // with H_i0+1 (columns 128-255).
  const int wq = warp & 3, ch2 = warp >> 2;
  const int r = 32 * wq + lane;
  const int half = wq >> 1;
  const int i = i0 + half;
  const int t = i * 64 + (r & 63);
  const bool valid = (i < nB) && (t < N);
  if (ok && (i < nB)) {  // warp-uniform
    const float inv = 1.f / (dpart[r] + dpart[128 + r]);
    __nv_bfloat16* dst = Ol + (static_cast<size_t>(bh) * N + (valid ? t : 0)) * kHeadDim + 64 * ch2;
#pragma unroll
    for (int cchunk = 0; cchunk < 2; ++cchunk) {
      uint32_t rr[32];
      tmem_ld32_sync(taddr + (static_cast<uint32_t>(32 * wq) << 16) + 128 * half + 64 * ch2 + 32 * cchunk, rr);
      if (valid) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * cchunk);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq)
          d4[qq] = make_uint4(
              pack_bf16x2(__uint_as_float(rr[8 * qq]) * inv, __uint_as_float(rr[8 * qq + 1]) * inv),
              pack_bf16x2(__uint_as_float(rr[8 * qq + 2]) * inv, __uint_as_float(rr[8 * qq + 3]) * inv),
              pack_bf16x2(__uint_as_float(rr[8 * qq + 4]) * inv, __uint_as_float(rr[8 * qq + 5]) * inv),
              pack_bf16x2(__uint_as_float(rr[8 * qq + 6]) * inv, __uint_as_float(rr[8 * qq + 7]) * inv));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(taddr, 256);
}

}  // namespace

cudaError_t launch_linear(const Dims& g, const void* q, float sm_scale, const void* mask,
                          const int32_t* marg, int m, const void* h, const float* z, char* ws,
                          cudaStream_t st) {
  if (m == 0) return cudaSuccess;
  const WsLayout L = ws_layout(g);
  int* status = reinterpret_cast<int*>(ws + L.status);
  __nv_bfloat16* Hbuf = reinterpret_cast<__nv_bfloat16*>(ws + L.Hbuf);
  float* Zbuf = reinterpret_cast<float*>(ws + L.Zbuf);
  __nv_bfloat16* Ol = reinterpret_cast<__nv_bfloat16*>(ws + L.Ol);

  CUtensorMap tmA, tmB, tmH;
  if (!make_tmap_3d(&tmA, mask, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.nBp, g.nB, g.BH, 64, 128) ||
      !make_tmap_3d(&tmB, h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kHeadDim * kHeadDim, g.nB, g.BH, 64,
                    64) ||
      !make_tmap_3d(&tmH, Hbuf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kHeadDim,
                    static_cast<uint64_t>(g.nB) * kHeadDim, g.BH, 64, 128))
    return cudaErrorInvalidValue;

  cudaError_t e = cudaFuncSetAttribute(hgemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(linout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kLinSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(zsum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kZSmem);
  if (e != cudaSuccess) return e;

  {
    TraceScope ts_("hgemm_kernel", st);
    hgemm_kernel<<<dim3(kHeadDim * kHeadDim / 128, (g.nB + 127) / 128, g.BH), 128, kGemmSmem, st>>>(
      tmA, tmB, Hbuf, g.nB, status);
  }
  {
    TraceScope ts_("zsum_kernel", st);
    zsum_kernel<<<dim3((g.nB + kZRows - 1) / kZRows, g.BH), 256, kZSmem, st>>>(
      z, static_cast<const __nv_bfloat16*>(mask), Zbuf, g.nB, g.nBp);
  }
  {
    TraceScope ts_("linout_kernel", st);
    linout_kernel<<<dim3((g.nB + 1) / 2, g.BH), kLinThreads, kLinSmem, st>>>(
      tmH, static_cast<const __nv_bfloat16*>(q), Zbuf, sm_scale, Ol, g.N, g.nB, status);
  }
  return cudaGetLastError();
}

}  // namespace sgs
