// backward.cu - gradients of the SageSLA output (dQ, dK, dV) for an upstream gradient dO.
//
// Method: "TurboDiffusion Demystified", section "Pillar Two: Sparse-Linear Attention - SLA"
// (the sparse-linear attention is trainable) and section "Advanced Guide: How is
// TurboDiffusion Trained?". The pages give no gradient; the one computed here is that of the
// forward definition with the block lists held fixed (they are discrete) and the INT8
// quantization read as the identity (straight through): scores Q~.K~^T in full precision,
// P not rounded by the method. Per (batch, head), with Q~ = c_s Q and K~ = K - mean_t K:
//   softmax branch over each query block's critical key blocks:
//     P = softmax(Q~ K~^T), O_s = P V, D = rowsum(dO o O_s), dS = P o (dO V^T - D),
//     dQ~ += dS K~, dK~ += dS^T Q~, dV += P^T dO;
//   linear branch over the marginal blocks (phi(x) = elu(x) + 1), per query block i with
//   H_i = sum_marg h_j, Z_i = sum_marg z_j and n = phi(Q~) H_i, den = phi(Q~) . Z_i:
//     dn = dO / den, dden = -(dO . O_l) / den, dphi(Q~) = dn H_i^T + dden Z_i^T,
//     dH_i = phi(Q~)^T dn, dZ_i = phi(Q~)^T dden, G_j = sum_{i: j marginal for i} dH_i,
//     g_j likewise, dV += phi(K~_j) G_j, dphi(K~_j) = V_j G_j^T + g_j;
//   dQ = c_s dQ~; dK = dK~ - mean_t dK~ (the smoothing mean depends on all of K).
//
// Kernels (bf16 operands, fp32 accumulation on the mma.sync m16n8k16 tensor-core path;
// 64-token blocks, four warps of 16 rows each):
//   tilde_kernel   Q~ and K~ rounded to bf16 once, so that the loops below stream raw tiles
//                  (cp.async into two buffers: the next tile's copy overlaps this one's math).
//   bwd_q_kernel   per query block: a statistics pass over the critical blocks (online
//                  softmax: O_s, LSE, D), a dQ pass, and the linear branch's dQ, dH_i, dZ_i.
//   (mask GEMM)    H = M h, Z = M z before, and G = M^T dH, g = M^T dZ after bwd_q_kernel
//                  (the forward's persistent tcgen05 GEMM, with the transposed mask).
//   bwd_kv_kernel  per key block, over the query blocks that hold it critical: dV, dK~, and
//                  the linear branch's dV and dK~ terms.
//   dk_mean / dk_sub  the token mean of dK~ in a fixed order, subtracted.
#include <math.h>

#include "../../include/sagesla.h"
#include "sagesla_internal.h"
#include "sm100_primitives.cuh"

namespace sgs {
namespace bwd {

constexpr int kLd = 136;                 // shared row stride in bf16 elements (272 B, conflict-free)
constexpr int kTileElems = 64 * kLd;     // one 64 x 128 tile
constexpr int kThreads = 128;
// Six 64 x 128 tiles: two fixed ones and two double-buffered pairs (the last pair of tiles
// also holds the 128-row H_i or G_j of the linear branch once the loops are done).
constexpr int kQSmem = 6 * kTileElems * 2 + (64 + 64 + 128 + 64) * 4;
constexpr int kKVSmem = 6 * kTileElems * 2 + (2 * 64 + 2 * 64 + 128) * 4;

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* qt;  // bf16(fl32(Q c_s)), [BH, N, d]
  const __nv_bfloat16* kt;  // bf16(fl32(K - mu)), [BH, N, d]
  const __nv_bfloat16* v;
  const __nv_bfloat16* dout;
  const float* k_mean;
  float c_s;
  const int32_t* crit;
  int k_c, m;
  const __nv_bfloat16* H;  // [BH, nB, d, d]
  const float* Z;          // [BH, nB, d]
  float* lse;              // [BH, Npad]
  float* dd;               // [BH, Npad]
  __nv_bfloat16* dH;       // [BH, nB, d, d]
  float* dZ;               // [BH, nB, d]
  const __nv_bfloat16* G;  // [BH, nB, d, d]
  const float* gz;         // [BH, nB, d]
  const uint32_t* cbits;   // [BH, nB, nW]: bit i of row j set when key block j is critical for i
  int nW;
  float* dq;
  float* dk;
  float* dv;
  float* kpart;            // [BH, nB, d]
  int N, nB, Npad;
};

// ---------------------------------------------------------------- mma.sync helpers
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// c += a (16x16, row) * b (16x8, col); bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Fragment addresses in a tile with row stride kLd (bf16). A 16x16 at (row r0, col c0),
// stored [m][k]: registers a0..a3 in mma order.
__device__ __forceinline__ uint32_t a_addr(uint32_t base, int r0, int c0, int lane) {
  return base + static_cast<uint32_t>(((r0 + (lane & 15)) * kLd + c0 + ((lane >> 4) << 3)) * 2);
}
// A 16x16 (m0.., k0..) from a tile stored [k][m]: a0..a3.
__device__ __forceinline__ uint32_t at_addr(uint32_t base, int k0, int m0, int lane) {
  return base + static_cast<uint32_t>(
                    ((k0 + (lane & 7) + (((lane >> 4) & 1) << 3)) * kLd + m0 + (((lane >> 3) & 1) << 3)) * 2);
}
// B for two n-tiles (n0..n0+15) x k16 (k0..) from a tile stored [n][k]:
// r0, r1 = b0, b1 of n-tile n0; r2, r3 = b0, b1 of n-tile n0+8.
__device__ __forceinline__ uint32_t bn_addr(uint32_t base, int n0, int k0, int lane) {
  return base + static_cast<uint32_t>(
                    ((n0 + (lane & 7) + ((lane >> 4) << 3)) * kLd + k0 + (((lane >> 3) & 1) << 3)) * 2);
}
// The same from a tile stored [k][n].
__device__ __forceinline__ uint32_t bt_addr(uint32_t base, int k0, int n0, int lane) {
  return base + static_cast<uint32_t>(
                    ((k0 + (lane & 7) + (((lane >> 3) & 1) << 3)) * kLd + n0 + ((lane >> 4) << 3)) * 2);
}
// Two C-layout 16x8 tiles (columns 16p..16p+15) packed as one bf16 A fragment.
__device__ __forceinline__ void c_to_a(const float (&c0)[4], const float (&c1)[4], uint32_t (&a)[4]) {
  a[0] = pack_bf16x2(c0[0], c0[1]);
  a[1] = pack_bf16x2(c0[2], c0[3]);
  a[2] = pack_bf16x2(c1[0], c1[1]);
  a[3] = pack_bf16x2(c1[2], c1[3]);
}

__device__ __forceinline__ float phi(float x) { return x > 0.f ? __fadd_rn(x, 1.f) : __expf(x); }
__device__ __forceinline__ float dphi(float x) { return x > 0.f ? 1.f : __expf(x); }

// Load rows [64*blk, 64*blk + 64) of one head's [N, 128] bf16 tensor into a shared tile,
// transformed, rounded to bf16; rows past N are zero.
// MODE 0: copy; 1: Q~ = fl32(x c_s); 2: K~ = fl32(x - mu); 3: phi(Q~); 4: phi(K~).
template <int MODE>
__device__ __forceinline__ void load_tile(__nv_bfloat16* dst, const __nv_bfloat16* src, int blk, int N,
                                          float c_s, const float* mu) {
  for (int x = threadIdx.x; x < 64 * 16; x += blockDim.x) {
    const int r = x >> 4, c8 = (x & 15) * 8;
    const int tok = blk * 64 + r;
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (tok < N) {
      u = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(tok) * kHeadDim + c8);
      if (MODE != 0) {
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w[e]));
          float a = f.x, b = f.y;
          if (MODE == 1 || MODE == 3) {
            a = __fmul_rn(a, c_s);
            b = __fmul_rn(b, c_s);
          } else {
            a = __fsub_rn(a, mu[c8 + 2 * e]);
            b = __fsub_rn(b, mu[c8 + 2 * e + 1]);
          }
          if (MODE >= 3) {
            a = phi(a);
            b = phi(b);
          }
          w[e] = pack_bf16x2(a, b);
        }
        u = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    *reinterpret_cast<uint4*>(dst + r * kLd + c8) = u;
  }
}

// ---- asynchronous tile copies (cp.async, 16 B per thread; a zero-byte source fills zeros)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}
// Rows [64*blk, 64*blk + 64) of one head's [N, 128] bf16 tensor, as stored, into a padded
// shared tile; rows past N are zero.
__device__ __forceinline__ void issue_tile(uint32_t dst, const __nv_bfloat16* src, int blk, int N) {
  for (int x = threadIdx.x; x < 64 * 16; x += blockDim.x) {
    const int r = x >> 4, c8 = (x & 15) * 8;
    const int tok = blk * 64 + r;
    const bool in = tok < N;
    cp_async16(dst + static_cast<uint32_t>((r * kLd + c8) * 2),
               src + static_cast<size_t>(in ? tok : 0) * kHeadDim + c8, in ? 16u : 0u);
  }
}

__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}
__device__ __forceinline__ float quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
}

// S (16 x 64 per warp) = A (16 x 128, from tile aA rows r0..) times B^T (B: 64 x 128 tile aB).
__device__ __forceinline__ void gemm_16x64_k128(float (&s)[8][4], uint32_t aA, int r0, uint32_t aB,
                                                int lane) {
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    uint32_t a[4];
    ldsm_x4(a_addr(aA, r0, 16 * kk, lane), a);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b[4];
      ldsm_x4(bn_addr(aB, 16 * np, 16 * kk, lane), b);
      mma16816(s[2 * np], a, b[0], b[1]);
      mma16816(s[2 * np + 1], a, b[2], b[3]);
    }
  }
}
// acc (16 x 128) += P (16 x 64, C layout in registers) times B (64 x 128 tile stored [k][n]).
__device__ __forceinline__ void gemm_acc_16x128_k64(float (&acc)[16][4], const float (&pc)[8][4],
                                                    uint32_t aB, int lane) {
#pragma unroll
  for (int kp = 0; kp < 4; ++kp) {
    uint32_t a[4];
    c_to_a(pc[2 * kp], pc[2 * kp + 1], a);
#pragma unroll
    for (int dp = 0; dp < 8; ++dp) {
      uint32_t b[4];
      ldsm_x4_t(bt_addr(aB, 16 * kp, 16 * dp, lane), b);
      mma16816(acc[2 * dp], a, b[0], b[1]);
      mma16816(acc[2 * dp + 1], a, b[2], b[3]);
    }
  }
}

// ---------------------------------------------------------------- dQ side
__global__ void __launch_bounds__(kThreads) bwd_q_kernel(Params p) {
  extern __shared__ __align__(16) unsigned char sm[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(sm);  // Q~ of block i
  __nv_bfloat16* sO = sQ + kTileElems;                        // dO of block i
  __nv_bfloat16* sK = sO + kTileElems;                        // K~_j / V_j buffer 0, later phi(Q~)
  __nv_bfloat16* sV = sK + kTileElems;                        //   and dn
  __nv_bfloat16* sH = sV + kTileElems;                        // K~_j / V_j buffer 1, later H_i [128][kLd]
  float* sDen = reinterpret_cast<float*>(sH + 128 * kLd);     // [64]
  float* sDd = sDen + 64;                                     // dden [64]
  float* sZ = sDd + 64;                                       // Z_i [128]
  float* sPart = sZ + 128;                                    // den partials [64]
  const int i = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
  const int r0 = 16 * warp;
  const size_t head = static_cast<size_t>(bh) * p.N * kHeadDim;
  const float* mu = p.k_mean + static_cast<size_t>(bh) * kHeadDim;
  const uint32_t aQ = smem_u32(sQ), aO = smem_u32(sO), aK = smem_u32(sK), aV = smem_u32(sV),
                 aH = smem_u32(sH);
  const int32_t* crit = p.crit + (static_cast<size_t>(bh) * p.nB + i) * p.k_c;
  const int rowA = i * 64 + r0 + g, rowB = rowA + 8;  // this thread's two query rows
  // K~_j and V_j of the walk's step jj go to buffer jj & 1 (tiles 2-3 or 4-5); the copies
  // of step jj + 1 run while step jj computes.
  auto issue_kv = [&](int jj) {
    const int j = __ldg(crit + jj);
    const uint32_t base = aK + static_cast<uint32_t>((jj & 1) * 2 * kTileElems * 2);
    issue_tile(base, p.kt + head, j, p.N);
    issue_tile(base + kTileElems * 2, p.v + head, j, p.N);
    cp_async_commit();
  };
  issue_tile(aQ, p.qt + head, i, p.N);
  issue_tile(aO, p.dout + head, i, p.N);
  issue_kv(0);  // one group with Q~ and dO

  // ---- pass 1: online softmax over the critical blocks -> O_s, LSE, D
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  float o[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  for (int jj = 0; jj < p.k_c; ++jj) {
    const int j = __ldg(crit + jj);
    if (jj + 1 < p.k_c) {
      issue_kv(jj + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t aKj = aK + static_cast<uint32_t>((jj & 1) * 2 * kTileElems * 2), aVj = aKj + kTileElems * 2;
    float s[8][4];
    gemm_16x64_k128(s, aQ, r0, aKj, lane);
    const int nvalid = min(64, p.N - j * 64);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (8 * nt + 2 * t4 + (e & 1) >= nvalid) s[nt][e] = -INFINITY;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * h], s[nt][2 * h + 1]));
      mx = quad_max(mx);
      const float mnew = fmaxf(mrow[h], mx);
      const float alpha = (mrow[h] == -INFINITY) ? 0.f : __expf(mrow[h] - mnew);
      float sum = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        s[nt][2 * h] = __expf(s[nt][2 * h] - mnew);
        s[nt][2 * h + 1] = __expf(s[nt][2 * h + 1] - mnew);
        sum += s[nt][2 * h] + s[nt][2 * h + 1];
      }
      lrow[h] = lrow[h] * alpha + sum;
      mrow[h] = mnew;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        o[nt][2 * h] *= alpha;
        o[nt][2 * h + 1] *= alpha;
      }
    }
    gemm_acc_16x128_k64(o, s, aVj, lane);
    __syncthreads();  // buffer jj & 1 is free for step jj + 2
  }
  float lse[2], dd[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float l = quad_sum(lrow[h]);
    lse[h] = mrow[h] + __logf(l);
    const float inv = 1.f / l;
    const int r = r0 + g + 8 * h;
    float acc = 0.f;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        acc += __bfloat162float(sO[r * kLd + 8 * nt + 2 * t4 + e]) * (o[nt][2 * h + e] * inv);
    dd[h] = quad_sum(acc);
  }
  if (t4 == 0) {
    const size_t base = static_cast<size_t>(bh) * p.Npad;
    p.lse[base + rowA] = rowA < p.N ? lse[0] : INFINITY;
    p.lse[base + rowB] = rowB < p.N ? lse[1] : INFINITY;
    p.dd[base + rowA] = rowA < p.N ? dd[0] : 0.f;
    p.dd[base + rowB] = rowB < p.N ? dd[1] : 0.f;
  }

  // ---- pass 2: dQ~ = sum_j dS K~_j, dS = P o (dO V^T - D)
  float dq[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) dq[nt][0] = dq[nt][1] = dq[nt][2] = dq[nt][3] = 0.f;
  issue_kv(0);
  for (int jj = 0; jj < p.k_c; ++jj) {
    const int j = __ldg(crit + jj);
    if (jj + 1 < p.k_c) {
      issue_kv(jj + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t aKj = aK + static_cast<uint32_t>((jj & 1) * 2 * kTileElems * 2), aVj = aKj + kTileElems * 2;
    float s[8][4], dp[8][4];
    gemm_16x64_k128(s, aQ, r0, aKj, lane);
    gemm_16x64_k128(dp, aO, r0, aVj, lane);
    const int nvalid = min(64, p.N - j * 64);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = e >> 1;
        const float pr = (8 * nt + 2 * t4 + (e & 1) < nvalid) ? __expf(s[nt][e] - lse[h]) : 0.f;
        s[nt][e] = pr * (dp[nt][e] - dd[h]);  // dS
      }
    gemm_acc_16x128_k64(dq, s, aKj, lane);
    __syncthreads();  // buffer jj & 1 is free for step jj + 2
  }

  // ---- linear branch: dQ~ += dphi o phi'(Q~); dH_i, dZ_i
  if (p.m > 0) {
    __syncthreads();
    load_tile<3>(sK, p.q + head, i, p.N, p.c_s, mu);  // phi(Q~), zero rows past N
    const __nv_bfloat16* Hi = p.H + (static_cast<size_t>(bh) * p.nB + i) * kHeadDim * kHeadDim;
    for (int x = threadIdx.x; x < 128 * 16; x += blockDim.x) {
      const int r = x >> 4, c8 = (x & 15) * 8;
      *reinterpret_cast<uint4*>(sH + r * kLd + c8) =
          *reinterpret_cast<const uint4*>(Hi + static_cast<size_t>(r) * kHeadDim + c8);
    }
    sZ[threadIdx.x] = p.Z[(static_cast<size_t>(bh) * p.nB + i) * kHeadDim + threadIdx.x];
    __syncthreads();
    {  // den = phi(Q~) . Z_i per row (two threads per row, 64 channels each)
      const int r = threadIdx.x >> 1, c0 = 64 * (threadIdx.x & 1);
      float acc = 0.f;
      for (int c = 0; c < 64; ++c) acc += __bfloat162float(sK[r * kLd + c0 + c]) * sZ[c0 + c];
      if (threadIdx.x & 1) sPart[r] = acc;
      __syncthreads();
      if (!(threadIdx.x & 1)) sDen[r] = acc + sPart[r];
      __syncthreads();
    }
    float nn[16][4];  // n = phi(Q~) H_i, then dn
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) nn[nt][0] = nn[nt][1] = nn[nt][2] = nn[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a[4];
      ldsm_x4(a_addr(aK, r0, 16 * kk, lane), a);
#pragma unroll
      for (int ep = 0; ep < 8; ++ep) {
        uint32_t b[4];
        ldsm_x4_t(bt_addr(aH, 16 * kk, 16 * ep, lane), b);
        mma16816(nn[2 * ep], a, b[0], b[1]);
        mma16816(nn[2 * ep + 1], a, b[2], b[3]);
      }
    }
    float dden[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = r0 + g + 8 * h;
      const bool valid = (i * 64 + r) < p.N;
      const float den = sDen[r];
      const float inv = valid ? 1.f / den : 0.f;
      float acc = 0.f;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float go = __bfloat162float(sO[r * kLd + 8 * nt + 2 * t4 + e]);
          acc += go * (nn[nt][2 * h + e] * inv);  // dO . O_l
          nn[nt][2 * h + e] = go * inv;           // dn
        }
      dden[h] = -quad_sum(acc) * inv;
    }
    // dphi(Q~) = dn H_i^T + dden Z_i^T
    float dph[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) dph[nt][0] = dph[nt][1] = dph[nt][2] = dph[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a[4];
      c_to_a(nn[2 * kk], nn[2 * kk + 1], a);
#pragma unroll
      for (int cp = 0; cp < 8; ++cp) {
        uint32_t b[4];
        ldsm_x4(bn_addr(aH, 16 * cp, 16 * kk, lane), b);
        mma16816(dph[2 * cp], a, b[0], b[1]);
        mma16816(dph[2 * cp + 1], a, b[2], b[3]);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = h ? rowB : rowA;
      const bool valid = row < p.N;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = 8 * nt + 2 * t4 + e;
          if (valid) {
            const float x = __fmul_rn(__bfloat162float(p.q[head + static_cast<size_t>(row) * kHeadDim + c]), p.c_s);
            dq[nt][2 * h + e] += (dph[nt][2 * h + e] + dden[h] * sZ[c]) * dphi(x);
          }
        }
    }
    // dn (bf16) and dden to shared memory for dH_i = phi(Q~)^T dn and dZ_i = phi(Q~)^T dden
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = r0 + g + 8 * h;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
        *reinterpret_cast<uint32_t*>(sV + r * kLd + 8 * nt + 2 * t4) =
            pack_bf16x2(nn[nt][2 * h], nn[nt][2 * h + 1]);
      if (t4 == 0) sDd[r] = dden[h];
    }
    __syncthreads();
    __nv_bfloat16* dHi = p.dH + (static_cast<size_t>(bh) * p.nB + i) * kHeadDim * kHeadDim;
#pragma unroll 1
    for (int eh = 0; eh < 2; ++eh) {
      float acc[2][8][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
#pragma unroll
      for (int kr = 0; kr < 4; ++kr) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          uint32_t a[4];
          ldsm_x4_t(at_addr(aK, 16 * kr, 32 * warp + 16 * mt, lane), a);
#pragma unroll
          for (int ep = 0; ep < 4; ++ep) {
            uint32_t b[4];
            ldsm_x4_t(bt_addr(aV, 16 * kr, 64 * eh + 16 * ep, lane), b);
            mma16816(acc[mt][2 * ep], a, b[0], b[1]);
            mma16816(acc[mt][2 * ep + 1], a, b[2], b[3]);
          }
        }
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c = 32 * warp + 16 * mt + g + 8 * h;
            const int e = 64 * eh + 8 * nt + 2 * t4;
            *reinterpret_cast<uint32_t*>(dHi + static_cast<size_t>(c) * kHeadDim + e) =
                pack_bf16x2(acc[mt][nt][2 * h], acc[mt][nt][2 * h + 1]);
          }
    }
    {  // dZ_i[c] = sum over rows of phi(Q~)[row][c] dden[row], rows in order
      const int c = threadIdx.x;
      float acc = 0.f;
      for (int r = 0; r < 64; ++r) acc = fmaf(__bfloat162float(sK[r * kLd + c]), sDd[r], acc);
      p.dZ[(static_cast<size_t>(bh) * p.nB + i) * kHeadDim + c] = acc;
    }
  }
  // dQ = c_s dQ~
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = h ? rowB : rowA;
    if (row < p.N) {
      float* dst = p.dq + head + static_cast<size_t>(row) * kHeadDim;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
        *reinterpret_cast<float2*>(dst + 8 * nt + 2 * t4) =
            make_float2(dq[nt][2 * h] * p.c_s, dq[nt][2 * h + 1] * p.c_s);
    }
  }
}

// ---------------------------------------------------------------- dK, dV side
__global__ void __launch_bounds__(kThreads) bwd_kv_kernel(Params p) {
  extern __shared__ __align__(16) unsigned char sm[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(sm);  // K~_j
  __nv_bfloat16* sV = sK + kTileElems;                        // V_j
  __nv_bfloat16* sQ = sV + kTileElems;                        // Q~_i / dO_i buffer 0, later phi(K~_j)
  __nv_bfloat16* sG = sQ + 2 * kTileElems;                    // Q~_i / dO_i buffer 1, later G_j [128][kLd]
  float* sLD = reinterpret_cast<float*>(sm + 6 * kTileElems * 2);  // [2 buffers][LSE_i 64 | D_i 64]
  float* sg = sLD + 2 * 128;                                        // g_j [128]
  const int j = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
  const int r0 = 16 * warp;
  const size_t head = static_cast<size_t>(bh) * p.N * kHeadDim;
  const float* mu = p.k_mean + static_cast<size_t>(bh) * kHeadDim;
  const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), aG = smem_u32(sG),
                 aLD = smem_u32(sLD);
  // Q~_i, dO_i, LSE_i and D_i of the n-th query block of the walk go to buffer n & 1; the
  // copies of the next block run while this one computes.
  auto issue_q = [&](int i, int buf) {
    const uint32_t base = aQ + static_cast<uint32_t>(buf * 2 * kTileElems * 2);
    issue_tile(base, p.qt + head, i, p.N);
    issue_tile(base + kTileElems * 2, p.dout + head, i, p.N);
    if (threadIdx.x < 32) {  // 2 x 256 B
      const size_t off = static_cast<size_t>(bh) * p.Npad + i * 64 + 4 * (threadIdx.x & 15);
      cp_async16(aLD + static_cast<uint32_t>((buf * 128 + 64 * (threadIdx.x >> 4) + 4 * (threadIdx.x & 15)) * 4),
                 ((threadIdx.x >> 4) ? p.dd : p.lse) + off, 16u);
    }
    cp_async_commit();
  };
  // the query blocks holding j critical, in increasing order (bits of cbits[bh][j])
  const uint32_t* bits = p.cbits + (static_cast<size_t>(bh) * p.nB + j) * p.nW;
  int w = 0;
  uint32_t word = p.nW > 0 ? __ldg(bits) : 0u;
  auto next_i = [&]() -> int {
    while (word == 0u) {
      if (++w >= p.nW) return -1;
      word = __ldg(bits + w);
    }
    const int i = 32 * w + __ffs(word) - 1;
    word &= word - 1;
    return i;
  };
  issue_tile(aK, p.kt + head, j, p.N);
  issue_tile(aV, p.v + head, j, p.N);
  int i_cur = next_i();
  if (i_cur >= 0) {
    issue_q(i_cur, 0);  // one group with K~_j and V_j
  } else {
    cp_async_commit();
  }
  float dk[16][4], dv[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    dk[nt][0] = dk[nt][1] = dk[nt][2] = dk[nt][3] = 0.f;
    dv[nt][0] = dv[nt][1] = dv[nt][2] = dv[nt][3] = 0.f;
  }
  for (int n = 0; i_cur >= 0; ++n) {
    const int i_nxt = next_i();
    if (i_nxt >= 0) {
      issue_q(i_nxt, (n + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int b = n & 1;
    const uint32_t aQi = aQ + static_cast<uint32_t>(b * 2 * kTileElems * 2), aOi = aQi + kTileElems * 2;
    const float* sL = sLD + b * 128;
    const float* sD = sL + 64;
    float st[8][4], dpt[8][4];
    gemm_16x64_k128(st, aK, r0, aQi, lane);   // S^T: keys x queries
    gemm_16x64_k128(dpt, aV, r0, aOi, lane);  // dP^T = V dO^T
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qc = 8 * nt + 2 * t4 + (e & 1);
        st[nt][e] = __expf(st[nt][e] - sL[qc]);           // P^T (0 for query rows past N)
        dpt[nt][e] = st[nt][e] * (dpt[nt][e] - sD[qc]);  // dS^T
      }
    gemm_acc_16x128_k64(dv, st, aOi, lane);   // dV += P^T dO
    gemm_acc_16x128_k64(dk, dpt, aQi, lane);  // dK~ += dS^T Q~
    __syncthreads();  // buffer n & 1 is free for block n + 2
    i_cur = i_nxt;
  }
  cp_async_wait<0>();
  __syncthreads();
  if (p.m > 0) {
    load_tile<4>(sQ, p.k + head, j, p.N, p.c_s, mu);  // phi(K~_j), zero rows past N
    const __nv_bfloat16* Gj = p.G + (static_cast<size_t>(bh) * p.nB + j) * kHeadDim * kHeadDim;
    for (int x = threadIdx.x; x < 128 * 16; x += blockDim.x) {
      const int r = x >> 4, c8 = (x & 15) * 8;
      *reinterpret_cast<uint4*>(sG + r * kLd + c8) =
          *reinterpret_cast<const uint4*>(Gj + static_cast<size_t>(r) * kHeadDim + c8);
    }
    sg[threadIdx.x] = p.gz[(static_cast<size_t>(bh) * p.nB + j) * kHeadDim + threadIdx.x];
    __syncthreads();
    // dV += phi(K~_j) G_j
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a[4];
      ldsm_x4(a_addr(aQ, r0, 16 * kk, lane), a);
#pragma unroll
      for (int ep = 0; ep < 8; ++ep) {
        uint32_t b[4];
        ldsm_x4_t(bt_addr(aG, 16 * kk, 16 * ep, lane), b);
        mma16816(dv[2 * ep], a, b[0], b[1]);
        mma16816(dv[2 * ep + 1], a, b[2], b[3]);
      }
    }
    // dphi(K~_j) = V_j G_j^T + g_j
    float dph[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) dph[nt][0] = dph[nt][1] = dph[nt][2] = dph[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a[4];
      ldsm_x4(a_addr(aV, r0, 16 * kk, lane), a);
#pragma unroll
      for (int cp = 0; cp < 8; ++cp) {
        uint32_t b[4];
        ldsm_x4(bn_addr(aG, 16 * cp, 16 * kk, lane), b);
        mma16816(dph[2 * cp], a, b[0], b[1]);
        mma16816(dph[2 * cp + 1], a, b[2], b[3]);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = j * 64 + r0 + g + 8 * h;
      if (row < p.N) {
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = 8 * nt + 2 * t4 + e;
            const float x = __fsub_rn(__bfloat162float(p.k[head + static_cast<size_t>(row) * kHeadDim + c]), mu[c]);
            dk[nt][2 * h + e] += (dph[nt][2 * h + e] + sg[c]) * dphi(x);
          }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = j * 64 + r0 + g + 8 * h;
    if (row < p.N) {
      float* dkr = p.dk + head + static_cast<size_t>(row) * kHeadDim;
      float* dvr = p.dv + head + static_cast<size_t>(row) * kHeadDim;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        *reinterpret_cast<float2*>(dkr + 8 * nt + 2 * t4) = make_float2(dk[nt][2 * h], dk[nt][2 * h + 1]);
        *reinterpret_cast<float2*>(dvr + 8 * nt + 2 * t4) = make_float2(dv[nt][2 * h], dv[nt][2 * h + 1]);
      }
    }
  }
  // this block's token sums of dK~ (rows in order), for the mean over tokens
  __syncthreads();
  {
    const int c = threadIdx.x;
    const int n = min(64, p.N - j * 64);
    float acc = 0.f;
    for (int r = 0; r < n; ++r) acc = __fadd_rn(acc, p.dk[head + static_cast<size_t>(j * 64 + r) * kHeadDim + c]);
    p.kpart[(static_cast<size_t>(bh) * p.nB + j) * kHeadDim + c] = acc;
  }
}

// Q~ = bf16(fl32(Q c_s)) and K~ = bf16(fl32(K - mu)), the operand tiles the two kernels
// stream (the same roundings a tile loader applying them on the fly would make).
__global__ void __launch_bounds__(256) tilde_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                    const float* __restrict__ k_mean, float c_s,
                                                    uint4* __restrict__ qt, uint4* __restrict__ kt,
                                                    size_t n8, int N) {
  for (size_t x = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; x < n8;
       x += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t bh = x / (static_cast<size_t>(N) * 16);
    const int c8 = static_cast<int>(x % 16) * 8;
    const float* mu = k_mean + bh * kHeadDim + c8;
    const uint4 uq = q[x], uk = k[x];
    uint32_t wq[4] = {uq.x, uq.y, uq.z, uq.w}, wk[4] = {uk.x, uk.y, uk.z, uk.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fq = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&wq[e]));
      const float2 fk = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&wk[e]));
      wq[e] = pack_bf16x2(__fmul_rn(fq.x, c_s), __fmul_rn(fq.y, c_s));
      wk[e] = pack_bf16x2(__fsub_rn(fk.x, mu[2 * e]), __fsub_rn(fk.y, mu[2 * e + 1]));
    }
    qt[x] = make_uint4(wq[0], wq[1], wq[2], wq[3]);
    kt[x] = make_uint4(wk[0], wk[1], wk[2], wk[3]);
  }
}

// Key block j is critical for query block i: bit i of cbits[bh][j].
__global__ void __launch_bounds__(64) crit_bits_kernel(const int32_t* __restrict__ crit, int nB, int k_c,
                                                       int nW, uint32_t* __restrict__ cbits) {
  const int i = blockIdx.x, bh = blockIdx.y;
  const int32_t* row = crit + (static_cast<size_t>(bh) * nB + i) * k_c;
  for (int x = threadIdx.x; x < k_c; x += blockDim.x) {
    const int j = __ldg(row + x);
    atomicOr(cbits + (static_cast<size_t>(bh) * nB + j) * nW + (i >> 5), 1u << (i & 31));
  }
}

// maskT[bh][j][i] = mask[bh][i][j] (bf16 0/1, row pitch nBp; the padding is left as zero).
__global__ void __launch_bounds__(256) mask_transpose_kernel(const __nv_bfloat16* __restrict__ mask,
                                                             __nv_bfloat16* __restrict__ maskT, int nB,
                                                             int nBp) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int bh = blockIdx.z, i0 = 32 * blockIdx.y, j0 = 32 * blockIdx.x;
  const size_t base = static_cast<size_t>(bh) * nB * nBp;
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int i = i0 + y, jj = j0 + threadIdx.x;
    tile[y][threadIdx.x] = (i < nB && jj < nB) ? mask[base + static_cast<size_t>(i) * nBp + jj]
                                               : __float2bfloat16(0.f);
  }
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int jj = j0 + y, i = i0 + threadIdx.x;
    if (jj < nB && i < nB) maskT[base + static_cast<size_t>(jj) * nBp + i] = tile[threadIdx.x][y];
  }
}

// mean[bh][c] = (sum over blocks of kpart, in block order) / N; dK = dK~ - mean.
__global__ void __launch_bounds__(128) dk_mean_kernel(const float* __restrict__ kpart, float* __restrict__ mean,
                                                      int nB, int N) {
  const int bh = blockIdx.x, c = threadIdx.x;
  float acc = 0.f;
  for (int j = 0; j < nB; ++j) acc = __fadd_rn(acc, kpart[(static_cast<size_t>(bh) * nB + j) * kHeadDim + c]);
  mean[bh * kHeadDim + c] = __fdiv_rn(acc, static_cast<float>(N));
}
__global__ void __launch_bounds__(256) dk_sub_kernel(float4* __restrict__ dk, const float* __restrict__ mean,
                                                     size_t n4, int N) {
  for (size_t x = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; x < n4;
       x += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t bh = x / (static_cast<size_t>(N) * 32);
    const int c = static_cast<int>(x % 32) * 4;
    const float* mrow = mean + bh * kHeadDim + c;
    float4 v = dk[x];
    v.x -= mrow[0];
    v.y -= mrow[1];
    v.z -= mrow[2];
    v.w -= mrow[3];
    dk[x] = v;
  }
}

}  // namespace bwd

// Workspace of the backward pass (byte offsets, 256-aligned).
struct BwdLayout {
  size_t status, H, Z, zb, lse, dd, dH, dZ, G, gz, maskT, cbits, kpart, kmean, qt, kt, total;
  int nW;
};
static size_t a256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
BwdLayout bwd_layout(const Dims& g) {
  BwdLayout L;
  const size_t BH = g.BH, nB = g.nB;
  L.nW = (g.nB + 31) / 32;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = a256(off + bytes);
    return o;
  };
  L.status = take(256);
  L.H = take(BH * nB * kHeadDim * kHeadDim * 2);
  L.Z = take(BH * nB * kHeadDim * 4);
  L.zb = take(BH * nB * kHeadDim * 2 * 2);
  L.lse = take(BH * g.Npad * 4);
  L.dd = take(BH * g.Npad * 4);
  L.dH = take(BH * nB * kHeadDim * kHeadDim * 2);
  L.dZ = take(BH * nB * kHeadDim * 4);
  L.G = take(BH * nB * kHeadDim * kHeadDim * 2);
  L.gz = take(BH * nB * kHeadDim * 4);
  L.maskT = take(BH * nB * g.nBp * 2);
  L.cbits = take(BH * nB * L.nW * 4);
  L.kpart = take(BH * nB * kHeadDim * 4);
  L.kmean = take(BH * kHeadDim * 4);
  L.qt = take(BH * g.N * kHeadDim * 2);
  L.kt = take(BH * g.N * kHeadDim * 2);
  L.total = off;
  return L;
}

size_t backward_workspace_bytes(const Dims& g) { return bwd_layout(g).total; }

cudaError_t launch_backward(const Dims& g, const void* q, const void* k, const void* v,
                            const void* dout, float sm_scale, const float* k_mean, const void* h,
                            const float* z, const int32_t* crit, int k_c, const void* mask, int m,
                            float* dq, float* dk, float* dv, char* ws, cudaStream_t st) {
  const BwdLayout L = bwd_layout(g);
  int* status = reinterpret_cast<int*>(ws + L.status);
  bwd::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.qt = reinterpret_cast<const __nv_bfloat16*>(ws + L.qt);
  p.kt = reinterpret_cast<const __nv_bfloat16*>(ws + L.kt);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.k_mean = k_mean;
  p.c_s = sm_scale;
  p.crit = crit;
  p.k_c = k_c;
  p.m = m;
  p.H = reinterpret_cast<const __nv_bfloat16*>(ws + L.H);
  p.Z = reinterpret_cast<const float*>(ws + L.Z);
  p.lse = reinterpret_cast<float*>(ws + L.lse);
  p.dd = reinterpret_cast<float*>(ws + L.dd);
  p.dH = reinterpret_cast<__nv_bfloat16*>(ws + L.dH);
  p.dZ = reinterpret_cast<float*>(ws + L.dZ);
  p.G = reinterpret_cast<const __nv_bfloat16*>(ws + L.G);
  p.gz = reinterpret_cast<const float*>(ws + L.gz);
  p.cbits = reinterpret_cast<const uint32_t*>(ws + L.cbits);
  p.nW = L.nW;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.kpart = reinterpret_cast<float*>(ws + L.kpart);
  p.N = g.N;
  p.nB = g.nB;
  p.Npad = g.Npad;
  __nv_bfloat16* zb = reinterpret_cast<__nv_bfloat16*>(ws + L.zb);
  cudaError_t e;
  if (m > 0) {  // H_i = sum_marg h_j, Z_i = sum_marg z_j (the forward's mask GEMM)
    e = launch_mask_gemm(g, mask, h, z, reinterpret_cast<__nv_bfloat16*>(ws + L.H),
                         reinterpret_cast<float*>(ws + L.Z), zb, status, st);
    if (e != cudaSuccess) return e;
  }
  {
    TraceScope ts_("tilde_kernel", st);
    const size_t n8 = static_cast<size_t>(g.BH) * g.N * 16;
    const int blocks = static_cast<int>((n8 + 255) / 256 < 8192 ? (n8 + 255) / 256 : 8192);
    bwd::tilde_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint4*>(q), static_cast<const uint4*>(k), k_mean,
                                              sm_scale, reinterpret_cast<uint4*>(ws + L.qt),
                                              reinterpret_cast<uint4*>(ws + L.kt), n8, g.N);
  }
  e = cudaFuncSetAttribute(bwd::bwd_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bwd::kQSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd::bwd_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bwd::kKVSmem);
  if (e != cudaSuccess) return e;
  {
    TraceScope ts_("bwd_q_kernel", st);
    bwd::bwd_q_kernel<<<dim3(g.nB, g.BH), bwd::kThreads, bwd::kQSmem, st>>>(p);
  }
  if (m > 0) {  // G_j = sum_{i: j marginal for i} dH_i, g_j likewise: the mask GEMM on M^T
    e = cudaMemsetAsync(ws + L.maskT, 0, static_cast<size_t>(g.BH) * g.nB * g.nBp * 2, st);
    if (e != cudaSuccess) return e;
    {
      TraceScope ts_("mask_transpose_kernel", st);
      bwd::mask_transpose_kernel<<<dim3((g.nB + 31) / 32, (g.nB + 31) / 32, g.BH), dim3(32, 8), 0, st>>>(
          static_cast<const __nv_bfloat16*>(mask), reinterpret_cast<__nv_bfloat16*>(ws + L.maskT), g.nB, g.nBp);
    }
    e = launch_mask_gemm(g, ws + L.maskT, ws + L.dH, reinterpret_cast<const float*>(ws + L.dZ),
                         reinterpret_cast<__nv_bfloat16*>(ws + L.G), reinterpret_cast<float*>(ws + L.gz), zb,
                         status, st);
    if (e != cudaSuccess) return e;
  }
  e = cudaMemsetAsync(ws + L.cbits, 0, static_cast<size_t>(g.BH) * g.nB * L.nW * 4, st);
  if (e != cudaSuccess) return e;
  {
    TraceScope ts_("crit_bits_kernel", st);
    bwd::crit_bits_kernel<<<dim3(g.nB, g.BH), 64, 0, st>>>(crit, g.nB, k_c, L.nW,
                                                           reinterpret_cast<uint32_t*>(ws + L.cbits));
  }
  {
    TraceScope ts_("bwd_kv_kernel", st);
    bwd::bwd_kv_kernel<<<dim3(g.nB, g.BH), bwd::kThreads, bwd::kKVSmem, st>>>(p);
  }
  {
    TraceScope ts_("dk_mean_kernel", st);
    bwd::dk_mean_kernel<<<g.BH, 128, 0, st>>>(p.kpart, reinterpret_cast<float*>(ws + L.kmean), g.nB, g.N);
  }
  {
    TraceScope ts_("dk_sub_kernel", st);
    const size_t n4 = static_cast<size_t>(g.BH) * g.N * 32;
    const int blocks = static_cast<int>((n4 + 255) / 256 < 8192 ? (n4 + 255) / 256 : 8192);
    bwd::dk_sub_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<float4*>(dk),
                                               reinterpret_cast<const float*>(ws + L.kmean), n4, g.N);
  }
  return cudaGetLastError();
}

}  // namespace sgs
