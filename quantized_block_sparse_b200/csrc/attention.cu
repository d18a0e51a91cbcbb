// attention.cu - block-sparse INT8 attention over the critical key blocks, merged with the
// linear-attention term of the marginal blocks.
//
// Method: "TurboDiffusion Demystified", section "Pillar One: Low-Bit Attention
// Acceleration - SageAttention" (Q K^T on INT8 tensor cores) and section "Pillar Two:
// Sparse-Linear Attention - SLA" (exact attention only on the selected block pairs; the
// two stack as "SageSLA").
//
// Design (sm_100a), two CTAs per SM:
//   * One CTA owns a PAIR of 64-row query blocks, i.e. one 128-row tile, so every
//     tensor-core instruction is a full M = 128 tcgen05.mma. pair_kernel chooses the
//     pairs: blocks sharing many critical key blocks go together. The CTA walks the union
//     of the two blocks' ascending critical lists; for a key block in only one list the
//     P.V MMA masks the other block's rows (disable-output-lane mask).
//   * The two blocks' rows are interleaved in 16-row groups (block i0 in TMEM lanes
//     32g..32g+15, block i1 in 32g+16..32g+31), so each block's softmax is spread over
//     all four SM sub-partitions, also on steps where only one block is critical.
//   * Warp-specialised:
//     - warp 0, TMA producer: the pair's Q8 once; per union step one INT8 K tile (8 KB)
//       into a 5-slot ring (with the step's block index, membership and k-scale beside
//       it) and one bf16 V tile (16 KB) into a 3-slot ring.
//     - warp 1, one thread issues every tcgen05.mma: kind::i8 S = Q8 K8^T (M128 N64 K128,
//       s32) into one of two 64-column TMEM score buffers, then kind::f16 O += P V with P
//       read from TMEM (M128 N128 K64, fp32 O in TMEM). QK(t+1) is issued before waiting
//       for P(t); P.V(t) as soon as the member halves have written P(t). Each tcgen05
//       instruction costs the issuing thread tens of cycles, so a step commits only twice:
//       once after QK (s_full) and once after P.V (the V slot's v_empty, which also tells
//       the rare rescale path that P.V has completed); the producer reuses a K slot once
//       its QK's s_full phase and the softmax warps' metadata reads (k_empty) are done.
//     - warps 2-9, softmax: two threads per query row (16-lane TMEM shapes, 16 keys each
//       of two rows), scores dequantised by s_q * s_k * log2(e) through an exact
//       magic-number int->float and packed f32x2 FMAs, exp2 on the SFU, P rounded to bf16
//       and written over the row's score columns.
//   * The running max m is raised only when a tile's partial sum of 2^(s - m) leaves
//     [0, 2^24]; only then is the exact tile max taken and O rescaled in TMEM.
//   * Linear branch (marginal blocks, when there are any): after a CTA's last step the
//     softmax warps write phi(Q~) of its 128 rows (recomputed from Q) as a K-major bf16
//     A tile over the Q8 tile and K slots 0-1, with each row's phi(Q~) . Z_i; the producer
//     streams H_i0 and H_i1 through the V ring as four 64 x 128 chunks; the MMA thread
//     forms phi(Q~) H_i in TMEM columns [0, 128) (freed by the last P.V), each block's
//     rows alone through the lane mask. O_l never goes to memory.
//   * Epilogue: O = O / l + (phi(Q~) H_i) / (phi(Q~) . Z_i) in fp32, rounded once to bf16.
// Every mbarrier wait is bounded (see sm100_primitives.cuh) and never traps.
#include <climits>

#include "sagesla_internal.h"
#include "sm100_primitives.cuh"

namespace sgs {
namespace {

constexpr int kPairWindow = 32;   // pairing: candidates per query block
constexpr int kPairSegment = 64;  // pairing: query blocks per segment (one CTA)

// K tiles (8 KB, read only by QK^T) and V tiles (16 KB, read by P.V after the softmax) sit
// in separate rings: a K slot frees as soon as its QK^T completes, so K runs far ahead;
// a V slot frees when its P.V completes.
constexpr int kKStages = 5;
constexpr int kVStages = 3;
constexpr int kKBytes = 8192;
constexpr int kVBytes = 16384;
constexpr int kOffQ = 0;
constexpr int kOffK = 16384;
constexpr int kOffV = kOffK + kKStages * kKBytes;
constexpr int kOffBar = kOffV + kVStages * kVBytes;
constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 8 + 4 + 1 + 1;
constexpr int kOffMeta = kOffBar + 512;               // per-K-slot tile metadata (StageMeta)
constexpr int kOffRowSum = kOffMeta + kKStages * 16;  // final row sums, [128]
constexpr int kOffDen = kOffRowSum + 128 * 4;          // linear-branch denominator halves, [2][128]
constexpr int kAttnSmem = kOffDen + 2 * 128 * 4 + 1024;  // ~107 KB: two CTAs per SM
// After the last Q K^T, the Q8 tile and K slots 0-1 ([0, 32 KB)) hold the phi(Q~) A tile of
// the linear branch: two 64-channel halves, 128 rows x 128 B each, K-major, 128-byte swizzle.
constexpr int kOffPhi = 0;
static_assert(kOffK + 2 * kKBytes == 32768 && kKStages >= 2, "phi(Q~) tile must fit over Q8 + 2 K slots");
static_assert(kNumBars * 8 + 4 <= kOffMeta - kOffBar, "barriers + TMEM slot overflow");
static_assert(2 * (kAttnSmem + 1024) <= 233472, "two CTAs per SM must fit in shared memory");
constexpr int kSoftmaxWarps = 8;
constexpr int kAttnThreads = 64 + 32 * kSoftmaxWarps;
constexpr float kLog2e = 1.4426950408889634f;
// The softmax reference point m of a row is raised only when a thread's partial sum of
// 2^(s - m) over its 16 keys of a tile exceeds 2^24 (or is not finite). Every accepted P is
// then <= 2^24, the row sum l <= 2^41 and O stays far from fp32 overflow; the exact tile
// max is computed only on that rare path (and on a row's first tile, where m = -inf).
constexpr float kPsumLimit = 16777216.0f;

// Written by the TMA producer for every union step next to its K tile, read by the MMA
// issuer and the softmax warps after they observe the slot's k_full phase (mbarrier
// release/acquire).
struct StageMeta {
  int j;       // key block
  int flags;   // bit 0: critical for the pair's first query block, bit 1: for the second,
               // bit 2: last step
  float sk;    // k_scale of block j
  int pad;
};

// TMEM columns: S0 [0,64), S1 [64,128) (int32 scores of one 128x64 tile; after the
// softmax, columns [0,32) of S_b hold the bf16 P tile, two values per column), O [128,256).
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 128;

struct AttnParams {
  const int2* pairs;       // [BH][nB]: (first, second) query block of each tile; -1 = none
  const int* pair_counts;  // [BH][n_seg]: tiles per segment of 64 query blocks
  const float* q_scale;
  const float* k_scale;
  const int32_t* crit;
  const __nv_bfloat16* q;   // bf16 Q [BH][N][d] (linear branch; nullptr when m == 0)
  const float* Z;           // Z_i fp32 [BH][nB][d]
  const __nv_bfloat16* H;   // H_i bf16 [BH][nB][d][d] (L2 prefetch only)
  float c_s;
  __nv_bfloat16* out;
  int* status;
  int N, nB, k_c, n_seg;
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

// ---- packed fp32 pairs (Blackwell f32x2 FMA / add: two lanes per instruction)
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

constexpr float kMagic = 12582912.f;  // 1.5 * 2^23
constexpr int kMagicBits = 0x4B400000;

// ---- TMEM access in the 16-lane shapes. For a 16-lane group starting at TMEM lane LB,
// thread t of the warp holds rows LB + t/4 and LB + t/4 + 8:
//   16x256b (8 columns per repetition k): regs 4k..4k+3 = (row0, 8k+2q), (row0, 8k+2q+1),
//           (row1, 8k+2q), (row1, 8k+2q+1) with q = t%4;
//   16x128b (4 columns per repetition k): regs 2k, 2k+1 = (row0, 4k+q), (row1, 4k+q).
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st_16x256b_x8(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_16x128b_x8(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// The softmax of one thread's share of a 64-key tile: rows row0/row1, 16 keys each (A: the
// exact floats 1.5*2^23 + int32 score in the 16x256b register order; the INT8 dot product
// over 128 channels is at most 128*127^2 < 2^22 in magnitude, so the integer is exact in the
// mantissa). P = 2^((A - 1.5*2^23)*sc - m_row), rounded to bf16 pairs in pk (16x128b order);
// returns the fp32 sums of this thread's P per row. Keys >= nvalid (a ragged last key block)
// get P = 0.
// FOLD: x = A*sc + (-m - 1.5*2^23*sc) in one FMA instead of (A - 1.5*2^23)*sc - m. The
// product is exact inside the FMA, so the only extra error is the rounding of the constant,
// at most half an ulp of 1.5*2^23*sc + m; callers fold only when 1.5*2^23*sc < 2^14, which
// bounds it by 2^-10 (log2 units; P within 0.07 %, below its own bf16 rounding). The error
// is common to a row's keys of one tile.
constexpr float kFoldLimit = 16384.f;
template <bool RAGGED, bool FOLD>
__device__ __forceinline__ void softmax_tile(const float (&A)[32], float sc, float negm0,
                                             float negm1, int q, int nvalid, uint32_t (&pk)[16],
                                             float& ps0, float& ps1) {
  const uint64_t sub = f2pack(-kMagic, -kMagic), sc2 = f2pack(sc, sc);
  const float msc = __fmul_rn(kMagic, sc);
  const float c0 = FOLD ? __fsub_rn(negm0, msc) : negm0, c1 = FOLD ? __fsub_rn(negm1, msc) : negm1;
  const uint64_t nm0 = f2pack(c0, c0), nm1 = f2pack(c1, c1);
  uint64_t acc0 = 0ull, acc1 = 0ull;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint64_t a01 = f2pack(A[4 * k], A[4 * k + 1]), a23 = f2pack(A[4 * k + 2], A[4 * k + 3]);
    const uint64_t x0 = fma2(FOLD ? a01 : add2(a01, sub), sc2, nm0);
    const uint64_t x1 = fma2(FOLD ? a23 : add2(a23, sub), sc2, nm1);
    float a0, a1, b0, b1, pa0, pa1, pb0, pb1;
    f2unpack(x0, a0, a1);
    f2unpack(x1, b0, b1);
    pa0 = ex2_approx(a0);
    pa1 = ex2_approx(a1);
    pb0 = ex2_approx(b0);
    pb1 = ex2_approx(b1);
    if (RAGGED) {
      const int c = 8 * k + 2 * q;
      if (c >= nvalid) pa0 = pb0 = 0.f;
      if (c + 1 >= nvalid) pa1 = pb1 = 0.f;
    }
    acc0 = add2(acc0, f2pack(pa0, pa1));
    acc1 = add2(acc1, f2pack(pb0, pb1));
    pk[2 * k] = pack_bf16x2(pa0, pa1);
    pk[2 * k + 1] = pack_bf16x2(pb0, pb1);
  }
  float a, b, c, d;
  f2unpack(acc0, a, b);
  f2unpack(acc1, c, d);
  ps0 = a + b;
  ps1 = c + d;
}

__device__ __forceinline__ float quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
}
__device__ __forceinline__ bool quad_any(bool v) {
  const unsigned bal = __ballot_sync(0xffffffffu, v);
  return ((bal >> ((threadIdx.x & 28u))) & 0xfu) != 0u;
}
__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}



// Same, with the disable-output-lane mask: bit k of the 128-bit mask (m0 = lanes 0-31, ...,
// m3 = lanes 96-127) keeps D lane k unchanged. Used for union steps that are critical for
// only one of the two query blocks.
__device__ __forceinline__ void mma_bf16_ts_masked(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                                   uint32_t idesc, uint32_t accumulate,
                                                   uint32_t m0, uint32_t m1, uint32_t m2,
                                                   uint32_t m3) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate), "r"(m0), "r"(m1), "r"(m2), "r"(m3));
}

// Both operands in shared memory, with the same disable-output-lane mask.
__device__ __forceinline__ void mma_bf16_ss_masked(uint32_t d_tmem, uint64_t a, uint64_t b,
                                                   uint32_t idesc, uint32_t accumulate,
                                                   uint32_t m0, uint32_t m1, uint32_t m2,
                                                   uint32_t m3) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(m0), "r"(m1), "r"(m2), "r"(m3));
}

__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmH,
                AttnParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + kKStages;
  uint64_t* v_full = k_empty + kKStages;
  uint64_t* v_empty = v_full + kVStages;
  // S ready for step t: s_full[t % 8], phase parity (t / 8) & 1. Eight barriers (for two
  // TMEM buffers) because a warp that skips steps (its half not critical) may reach step t
  // as early as the completion of QK(t-5) (the K ring depth); the barrier's previous phase,
  // step t-8, is then always complete, so a parity wait can never alias.
  uint64_t* s_full = v_empty + kVStages;
  uint64_t* p_full = s_full + 8;  // [half][buffer]
  uint64_t* o_full = p_full + 4;
  uint64_t* lsum_bar = o_full + 1;  // final row sums written (all softmax threads)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lsum_bar + 1);
  StageMeta* meta = reinterpret_cast<StageMeta*>(smem + kOffMeta);
  float* rowsum = reinterpret_cast<float*>(smem + kOffRowSum);
  float* denp = reinterpret_cast<float*>(smem + kOffDen);
  __shared__ int abort_flag;

  const int pr = blockIdx.x, bh = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nB = p.nB;
  // Tile pr of the head is entry `tile` of segment `seg`. Every warp finds it at once, with
  // one round of loads instead of a chain of dependent ones: lane l holds the tile counts of
  // segments 4l..4l+3 (n_seg <= 128), an inclusive warp scan of their sums gives each lane
  // its range of tiles, and the lane whose range holds pr walks its four segments.
  int tile = pr, seg = 0;
  {
    const int* cnt = p.pair_counts + static_cast<size_t>(bh) * p.n_seg;
    int c[4], own = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      c[u] = 4 * lane + u < p.n_seg ? __ldg(cnt + 4 * lane + u) : 0;
      own += c[u];
    }
    int incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, pr >= incl - own && pr < incl);
    if (hit == 0u) return;  // past the head's last tile (whole CTA, before any barrier)
    const int src = __ffs(hit) - 1;
    tile = pr - __shfl_sync(0xffffffffu, incl - own, src);
    seg = 4 * src;
    bool found = false;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int cu = __shfl_sync(0xffffffffu, c[u], src);
      if (!found) {
        if (tile < cu) {
          seg = 4 * src + u;
          found = true;
        } else {
          tile -= cu;
        }
      }
    }
  }
  const int2 pq = p.pairs[static_cast<size_t>(bh) * nB + seg * kPairSegment + tile];
  const int i0 = pq.x, i1 = pq.y;  // the pair (i1 = -1: block i0 alone)
  // Linear branch: H_i0 (and H_i1) enter the V ring after the last V tile as 16 KB chunks
  // of 64 channels x 128 columns: chunk u is rows [64*(u&1), +64) of H of block u>>1.
  const bool lin = p.q != nullptr;
  const int nH = lin ? (i1 >= 0 ? 4 : 2) : 0;

  UnionWalk walk;
  walk.c0 = p.crit + (static_cast<size_t>(bh) * nB + i0) * p.k_c;
  walk.c1 = p.crit + (static_cast<size_t>(bh) * nB + (i1 >= 0 ? i1 : i0)) * p.k_c;
  walk.n0 = p.k_c;
  walk.n1 = (i1 >= 0) ? p.k_c : 0;
  walk.p0 = 0;
  walk.p1 = 0;

  if (tid == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(smem_u32(k_full + s), 1);
      mbar_init(smem_u32(k_empty + s), kSoftmaxWarps);  // every softmax warp has read the metadata
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(smem_u32(v_full + s), 1);
      mbar_init(smem_u32(v_empty + s), 1);  // P.V commit
    }
    for (int x = 0; x < 8; ++x) mbar_init(smem_u32(s_full + x), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(p_full + b), 128);      // half 0 rows, buffer b
      mbar_init(smem_u32(p_full + 2 + b), 128);  // half 1 rows, buffer b
    }
    mbar_init(smem_u32(o_full), 1);
    mbar_init(smem_u32(lsum_bar), 32 * kSoftmaxWarps);
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    if (lin) prefetch_tmap(&tmH);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;
  const uint32_t sQ = smem_u32(smem + kOffQ);
  const uint32_t sK = smem_u32(smem + kOffK);
  const uint32_t sV = smem_u32(smem + kOffV);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // One thread feeds both rings without blocking on either: K tiles (with the step's
    // metadata) run up to kKStages steps ahead of the V tiles.
    if (lane == 0) {
      // rows interleaved in 16-row groups: tile rows 32g..32g+15 = block i0 rows 16g..16g+15,
      // tile rows 32g+16..32g+31 = block i1 rows 16g..16g+15 (TMEM lane = tile row)
      mbar_expect_tx(smem_u32(q_full), 16384);
      const int i1r = i1 >= 0 ? i1 : i0;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        tma_load_3d(sQ + 4096 * g, &tmQ, smem_u32(q_full), 0, i0 * 64 + 16 * g, bh);
        tma_load_3d(sQ + 4096 * g + 2048, &tmQ, smem_u32(q_full), 0, i1r * 64 + 16 * g, bh);
      }
      int j, fl;
      bool have = walk.next(j, fl);  // k_c >= 1: at least one step
      int tK = 0, tV = 0, nsteps = -1;  // nsteps: known once the walk is exhausted
      int ks = 0, kph = 0, vs = 0, vph = 0;
      unsigned long long t_idle = 0;
      for (;;) {
        bool progress = false;
        // K: as far ahead as the ring allows (and never more than kKStages beyond V)
        // a K slot is free once every softmax warp has read its metadata (k_empty) and the
        // QK^T of its previous step has completed (that step's s_full phase)
        while (have && tK < tV + kKStages &&
               (tK < kKStages ||
                (mbar_test_wait(smem_u32(k_empty + ks), kph ^ 1) &&
                 mbar_test_wait(smem_u32(s_full + ((tK - kKStages) & 7)), ((tK - kKStages) >> 3) & 1)))) {
          int jn, fln;
          const bool have_next = walk.next(jn, fln);
          meta[ks].j = j;
          meta[ks].flags = fl | (have_next ? 0 : 4);
          meta[ks].sk = __ldg(p.k_scale + static_cast<size_t>(bh) * nB + j);
          mbar_expect_tx(smem_u32(k_full + ks), kKBytes);
          tma_load_3d(sK + ks * kKBytes, &tmK, smem_u32(k_full + ks), 0, j * 64, bh);
          ++tK;
          if (++ks == kKStages) {
            ks = 0;
            kph ^= 1;
          }
          if (!have_next) {
            nsteps = tK;
            if (lin) {  // the linear branch's H tiles and Q rows, needed at the end of the walk
              for (int b = 0; b < (i1 >= 0 ? 2 : 1); ++b) {
                const int ib = b ? i1 : i0;
                prefetch_l2(p.H + (static_cast<size_t>(bh) * nB + ib) * (kHeadDim * kHeadDim),
                            kHeadDim * kHeadDim * 2);
                const int rows = min(64, p.N - ib * 64);
                prefetch_l2(p.q + (static_cast<size_t>(bh) * p.N + ib * 64) * kHeadDim,
                            static_cast<uint32_t>(rows) * kHeadDim * 2);
              }
            }
          }
          have = have_next;
          j = jn;
          fl = fln;
          progress = true;
        }
        // V: the next step whose K has been issued, once its slot is free; after the last
        // step, the linear branch's H chunks take the same ring
        const bool v_next = tV < tK || (nsteps >= 0 && tV < nsteps + nH);
        if (v_next && (tV < kVStages || mbar_test_wait(smem_u32(v_empty + vs), vph ^ 1))) {
          mbar_expect_tx(smem_u32(v_full + vs), kVBytes);
          if (tV < tK) {
            const int jv = meta[tV % kKStages].j;  // K slot of step tV: not reused before V(tV)
            tma_load_3d(sV + vs * kVBytes, &tmV, smem_u32(v_full + vs), 0, jv * 64, bh);
            tma_load_3d(sV + vs * kVBytes + 8192, &tmV, smem_u32(v_full + vs), 64, jv * 64, bh);
          } else {
            const int u = tV - nsteps;
            const int crow = ((u >> 1) ? i1 : i0) * kHeadDim + 64 * (u & 1);
            tma_load_3d(sV + vs * kVBytes, &tmH, smem_u32(v_full + vs), 0, crow, bh);
            tma_load_3d(sV + vs * kVBytes + 8192, &tmH, smem_u32(v_full + vs), 64, crow, bh);
          }
          ++tV;
          if (++vs == kVStages) {
            vs = 0;
            vph ^= 1;
          }
          progress = true;
        }
        if (nsteps >= 0 && tV == nsteps + nH) break;
        if (progress) {
          t_idle = 0;
          continue;
        }
        // nothing to issue: sleep on the V slot we need next (the usual blocker)
        if (v_next && tV >= kVStages) mbar_try_wait_suspend(smem_u32(v_empty + vs), vph ^ 1, 2000u);
        else if (tK >= kKStages) mbar_try_wait_suspend(smem_u32(k_empty + ks), kph ^ 1, 2000u);
        if (abort_flag) {
          break;
        }
        const unsigned long long now = globaltimer();
        if (t_idle == 0) {
          t_idle = now;
        } else if (now - t_idle > kWaitLimitNs) {
          abort_flag = 1;
          atomicOr(p.status, kStatusTimeout);
          break;
        }
      }
      {  // every copy issued lands before the CTA exits (already true unless a wait gave up)
        mbar_drain(smem_u32(q_full), 0, p.status);
        for (int u = max(0, tK - kKStages); u < tK; ++u)
          mbar_drain(smem_u32(k_full + (u % kKStages)), (u / kKStages) & 1, p.status);
        for (int u = max(0, tV - kVStages); u < tV; ++u)
          mbar_drain(smem_u32(v_full + (u % kVStages)), (u / kVStages) & 1, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order QK(0), QK(1), PV(0), QK(2), PV(1), ...: tcgen05.mma ops from one thread
    // execute in issue order, so QK(t) overwriting S_(t%2) (which holds P(t-2)) runs after
    // PV(t-2) has read it. PV waits only for the halves that are critical for its step and
    // masks the D lanes of the other half.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(2, 1, 0, 0, 128, 64);
      constexpr uint32_t idesc_pv = make_idesc(1, 1, 0, 1, 128, 128);
      const uint64_t dq = make_sdesc(sQ, 16, 1024);
      const uint64_t dk0 = make_sdesc(sK, 16, 1024);
      const uint64_t dv0 = make_sdesc(sV, 8192, 1024);
      constexpr uint64_t kKDesc = kKBytes >> 4;  // start-address field units (16 B)
      constexpr uint64_t kVDesc = kVBytes >> 4;
      bool ok = mbar_wait(smem_u32(q_full), 0, &abort_flag, p.status);
      int pcnt[2][2] = {{0, 0}, {0, 0}};  // completed p_full phases per (half, buffer)
      int prev_flags = 0;
      int vs = 0, vph = 0;
      auto issue_pv = [&](int u, int fl) -> bool {
        const int b = u & 1;
        if (!mbar_wait(smem_u32(v_full + vs), vph, &abort_flag, p.status)) return false;
        for (int h = 0; h < 2; ++h) {
          if (fl & (1 << h)) {
            if (!mbar_wait(smem_u32(p_full + 2 * h + b), pcnt[h][b] & 1, &abort_flag, p.status))
              return false;
            ++pcnt[h][b];
          }
        }
        tc_fence_after();
        // block i0 owns lanes 0-15 of every 32-lane group, block i1 lanes 16-31: a set bit
        // disables that output lane
        const uint32_t mk = ((fl & 1) ? 0u : 0x0000ffffu) | ((fl & 2) ? 0u : 0xffff0000u);
        const uint64_t dv = dv0 + kVDesc * vs;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts_masked(taddr + kColO, taddr + 64 * b + 8 * kk, dv + 128 * kk, idesc_pv, 1u,
                             mk, mk, mk, mk);
        mma_commit(smem_u32(v_empty + vs));  // V slot free, and P.V(u) complete (rescale)
        if (++vs == kVStages) {
          vs = 0;
          vph ^= 1;
        }
        return true;
      };
      int t = 0, s = 0, ph = 0;
      bool last = false;
      while (ok && !last) {
        const int b = t & 1;
        if (!mbar_wait(smem_u32(k_full + s), ph, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        const int fl = meta[s].flags;
        last = (fl & 4) != 0;
        tc_fence_after();
        const uint64_t dk = dk0 + kKDesc * s;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_i8(taddr + 64 * b, dq + 2 * kk, dk + 2 * kk, idesc_qk, kk > 0 ? 1u : 0u);
        mma_commit(smem_u32(s_full + (t & 7)));
        if (t >= 1 && !issue_pv(t - 1, prev_flags)) {
          ok = false;
          break;
        }
        prev_flags = fl;
        ++t;
        if (++s == kKStages) {
          s = 0;
          ph ^= 1;
        }
      }
      if (ok && t >= 1) ok = issue_pv(t - 1, prev_flags);
      if (ok && lin) {
        // Linear branch into TMEM columns [0, 128) (free once the last P.V has read P, which
        // issue order guarantees): phi(Q~) (written by the softmax warps, lsum_bar) times
        // the H chunks from the V ring, each block's rows alone (the other's lanes masked).
        ok = mbar_wait(smem_u32(lsum_bar), 0, &abort_flag, p.status);
        const uint64_t da = make_sdesc(smem_u32(smem + kOffPhi), 16, 1024);
        for (int u = 0; u < nH && ok; ++u) {
          if (!mbar_wait(smem_u32(v_full + vs), vph, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t mk = (u >> 1) ? 0x0000ffffu : 0xffff0000u;
          const uint64_t a = da + static_cast<uint64_t>((u & 1) * (16384 >> 4));
          const uint64_t dv = dv0 + kVDesc * vs;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss_masked(taddr, a + 2 * kk, dv + 128 * kk, idesc_pv, ((u & 1) | kk) != 0 ? 1u : 0u,
                               mk, mk, mk, mk);
          mma_commit(smem_u32(v_empty + vs));
          if (++vs == kVStages) {
            vs = 0;
            vph ^= 1;
          }
        }
      }
      mma_commit(smem_u32(o_full));
      mbar_drain(smem_u32(o_full), 0, p.status);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 2-9)
    // Warp w owns the 16 TMEM lanes LB = 32*(w%4) + 16*((w-2)/4) .. LB+15: rows 16*(w%4)..+15
    // of block i0 for warps 2-5 and of block i1 for warps 6-9 (interleaved layout), so
    // membership is warp-uniform. In the 16-lane load shape thread t holds rows LB + t/4
    // and LB + t/4 + 8, 16 keys each; the four threads of a quad (t/4) share rows. A warp
    // whose block is not critical for a step skips it (the P.V MMA masks its rows).
    const int wq = warp & 3;
    const int sub = (warp - 2) >> 2;
    const uint32_t lb = 32 * wq + 16 * sub;
    const int q = lane & 3;
    const int rr0 = static_cast<int>(lb) + (lane >> 2);  // rows rr0 and rr0 + 8
    const int half = sub;  // lanes 32*wq + 16*sub .. +15 hold rows of block i0 (sub 0) or i1
    const int i = half ? i1 : i0;
    const float sq = (i >= 0) ? p.q_scale[static_cast<size_t>(bh) * nB + i] : 0.f;
    const uint32_t lane_off = lb << 16;
    {  // O starts at zero for these rows; every P.V then accumulates
      uint32_t z[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) z[c] = 0u;
      tmem_st_16x256b_x8(taddr + lane_off + kColO, z);
      tmem_st_16x256b_x8(taddr + lane_off + kColO + 64, z);
      tmem_wait_st();
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool ok = true;
    bool last = false;
    int t = 0, s = 0, ph = 0;
    while (!last) {
      const int b = t & 1;
      ok = mbar_wait(smem_u32(k_full + s), ph, &abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      const int j = meta[s].j, fl = meta[s].flags;
      const float skj = meta[s].sk;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(k_empty + s));
      last = (fl & 4) != 0;
      const bool member = (fl >> half) & 1;  // warp-uniform
      if (member) {
        ok = mbar_wait(smem_u32(s_full + (t & 7)), (t >> 3) & 1, &abort_flag, p.status);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[32];
        tmem_ld_16x256b_x8(taddr + lane_off + 64 * b, sv);
        const bool ragged = (j == nB - 1) && (p.N - j * 64 < 64);  // CTA-uniform
        const int nvalid = ragged ? p.N - j * 64 : 64;
        float A[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) A[c] = __int_as_float(static_cast<int>(sv[c]) + kMagicBits);
        const float sc = __fmul_rn(__fmul_rn(sq, skj), kLog2e);
        uint32_t pk[16];
        float ps0, ps1;
        const bool fold = __fmul_rn(kMagic, sc) < kFoldLimit;  // warp-uniform
        auto run_tile = [&]() {
          if (ragged) {
            if (fold) softmax_tile<true, true>(A, sc, -m0, -m1, q, nvalid, pk, ps0, ps1);
            else softmax_tile<true, false>(A, sc, -m0, -m1, q, nvalid, pk, ps0, ps1);
          } else {
            if (fold) softmax_tile<false, true>(A, sc, -m0, -m1, q, 64, pk, ps0, ps1);
            else softmax_tile<false, false>(A, sc, -m0, -m1, q, 64, pk, ps0, ps1);
          }
        };
        run_tile();
        // rare path: raise m where a partial sum left [0, 2^24] (quad-consistent decision;
        // the warp-wide test first keeps the common path to one vote)
        float alpha0 = 1.f, alpha1 = 1.f;
        bool rescale = false;
        if (__any_sync(0xffffffffu, !(ps0 <= kPsumLimit) || !(ps1 <= kPsumLimit))) {
          const bool need0 = quad_any(!(ps0 <= kPsumLimit)), need1 = quad_any(!(ps1 <= kPsumLimit));
          // S_b still holds the scores (P overwrites it only below): reload them.
          tmem_ld_16x256b_x8(taddr + lane_off + 64 * b, sv);
#pragma unroll
          for (int c = 0; c < 32; ++c) A[c] = __int_as_float(static_cast<int>(sv[c]) + kMagicBits);
          float mA0 = 0.f, mA1 = 0.f;  // 0 is below every real value (all >= 1.5*2^23 - 2^22)
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int c = 8 * k + 2 * q;
            if (c < nvalid) {
              mA0 = fmaxf(mA0, A[4 * k]);
              mA1 = fmaxf(mA1, A[4 * k + 2]);
            }
            if (c + 1 < nvalid) {
              mA0 = fmaxf(mA0, A[4 * k + 1]);
              mA1 = fmaxf(mA1, A[4 * k + 3]);
            }
          }
          mA0 = quad_max(mA0);
          mA1 = quad_max(mA1);
          if (need0) {
            const float mt = __fmul_rn(__fsub_rn(mA0, kMagic), sc);
            if (m0 != -INFINITY) alpha0 = ex2_approx(m0 - mt);
            m0 = mt;
          }
          if (need1) {
            const float mt = __fmul_rn(__fsub_rn(mA1, kMagic), sc);
            if (m1 != -INFINITY) alpha1 = ex2_approx(m1 - mt);
            m1 = mt;
          }
          run_tile();
          rescale = __any_sync(0xffffffffu, alpha0 != 1.f || alpha1 != 1.f);
        }
        l0 = fmaf(l0, alpha0, ps0);
        l1 = fmaf(l1, alpha1, ps1);
        tmem_st_16x128b_x8(taddr + lane_off + 64 * b, pk);  // P first: its registers die here
        if (rescale) {  // warp-uniform
          // O holds P.V of earlier steps: wait for the last issued P.V, then rescale rows.
          if (t >= 1)  // P.V(t-1) complete: the v_empty phase of its V slot
            ok = mbar_wait(smem_u32(v_empty + ((t - 1) % kVStages)), ((t - 1) / kVStages) & 1,
                           &abort_flag, p.status);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {  // 2 x 64 columns of O (16x256b.x8 spans 64)
            uint32_t o[32];
            const uint32_t oa = taddr + lane_off + kColO + 64 * cc;
            tmem_ld_16x256b_x8(oa, o);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              o[4 * k] = __float_as_uint(__uint_as_float(o[4 * k]) * alpha0);
              o[4 * k + 1] = __float_as_uint(__uint_as_float(o[4 * k + 1]) * alpha0);
              o[4 * k + 2] = __float_as_uint(__uint_as_float(o[4 * k + 2]) * alpha1);
              o[4 * k + 3] = __float_as_uint(__uint_as_float(o[4 * k + 3]) * alpha1);
            }
            tmem_st_16x256b_x8(oa, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(p_full + 2 * half + b));
      }
      ++t;
      if (++s == kKStages) {
        s = 0;
        ph ^= 1;
      }
    }

    // ------------------------------------------------------------ epilogue
    // Row sums: quad reduce, then hand them to the one-row-per-thread epilogue layout.
    l0 = quad_sum(l0);
    l1 = quad_sum(l1);
    if (q == 0) {
      rowsum[rr0] = l0;
      rowsum[rr0 + 8] = l1;
    }
    // Epilogue layout: warp w reads its quadrant's 32 lanes (32x32b), one row per thread,
    // output columns [64*sub, 64*sub + 64).
    const int r = 32 * wq + lane;
    const int ie = (lane >> 4) ? i1 : i0;
    const int tok = ie * 64 + 16 * wq + (lane & 15);
    const bool row_valid = (ie >= 0) && (tok < p.N);
    if (lin && ok) {
      // phi(Q~) of this row's channels [64*sub, +64) into the A tile over Q8 and K slots 0-1,
      // free once every Q K^T has completed (the last step's S is ready), and this half of
      // the denominator phi(Q~).Z_i with the bf16-rounded phi the tensor core sees.
      if (t >= 1) ok = mbar_wait(smem_u32(s_full + ((t - 1) & 7)), ((t - 1) >> 3) & 1, &abort_flag, p.status);
      const uint32_t tile = smem_u32(smem + kOffPhi) + sub * 16384;
      float dacc = 0.f;
      if (row_valid) {
        const uint4* qr = reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(bh) * p.N + tok) * kHeadDim + 64 * sub);
        const float4* zr = reinterpret_cast<const float4*>(p.Z + (static_cast<size_t>(bh) * nB + ie) * kHeadDim + 64 * sub);
        uint4 qv[8];
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) qv[cb] = __ldg(qr + cb);
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) {
          const float4 z0 = __ldg(zr + 2 * cb), z1 = __ldg(zr + 2 * cb + 1);
          const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
          uint32_t w[4] = {qv[cb].x, qv[cb].y, qv[cb].z, qv[cb].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = __fmul_rn(__uint_as_float(w[e] << 16), p.c_s);
            const float x1 = __fmul_rn(__uint_as_float(w[e] & 0xffff0000u), p.c_s);
            w[e] = pack_bf16x2(x0 > 0.f ? x0 + 1.f : ex2_approx(x0 * kLog2e),
                               x1 > 0.f ? x1 + 1.f : ex2_approx(x1 * kLog2e));
            dacc = fmaf(__uint_as_float(w[e] << 16), zz[2 * e], dacc);
            dacc = fmaf(__uint_as_float(w[e] & 0xffff0000u), zz[2 * e + 1], dacc);
          }
          st_shared_v4(tile + sw128_offset(r, cb), w[0], w[1], w[2], w[3]);
        }
      } else {
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) st_shared_v4(tile + sw128_offset(r, cb), 0u, 0u, 0u, 0u);
      }
      denp[sub * 128 + r] = dacc;
      fence_async_smem();
    }
    mbar_arrive(smem_u32(lsum_bar));
    ok = ok && mbar_wait(smem_u32(lsum_bar), 0, &abort_flag, p.status);
    ok = ok && mbar_wait(smem_u32(o_full), 0, &abort_flag, p.status);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    const uint32_t eoff = static_cast<uint32_t>(32 * wq) << 16;
    if (ok) {
      // O = O_s / l + O_lin / den, one rounding to bf16
      const float inv = 1.f / rowsum[r];
      const float invd = lin ? 1.f / (denp[r] + denp[128 + r]) : 0.f;
      const size_t row = static_cast<size_t>(bh) * p.N + (row_valid ? tok : 0);
      __nv_bfloat16* dst = p.out + row * kHeadDim + 64 * sub;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t o[32], ol[32];
        tmem_ld32_sync(taddr + eoff + kColO + 64 * sub + 32 * cc, o);
        if (lin) tmem_ld32_sync(taddr + eoff + 64 * sub + 32 * cc, ol);
        if (row_valid) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * cc);
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              f[e] = fmaf(__uint_as_float(o[8 * qq + e]), inv, lin ? __uint_as_float(ol[8 * qq + e]) * invd : 0.f);
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

// Pairs of query blocks for the attention tiles. Two blocks that share many critical key
// blocks make a short union walk: the tile executes |crit(i0) U crit(i1)| steps for 2*k_c
// useful ones. One CTA per (head, segment of 64 query blocks): the segment's blocks are
// taken in ascending order and each unpaired block is matched with the unpaired block
// among the next 32 of the segment that shares the most critical blocks (ties: the
// nearest), or left alone. Segment s writes its n_s tiles, (i0, i1) with i1 = -1 for a
// block left alone, to pairs[bh][64*s + k] and n_s to counts[bh][s]; tile t of a head is
// then entry t - (n_0 + ... + n_{s-1}) of the segment s where that sum passes t.
__global__ void __launch_bounds__(256) pair_kernel(const int32_t* __restrict__ crit, int nB, int k_c,
                                                   int2* __restrict__ pairs, int* __restrict__ counts) {
  extern __shared__ uint32_t psm[];
  const int seg = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int lo = seg * kPairSegment, hi = min(nB, lo + kPairSegment), rows = hi - lo;
  const int nW = ((nB + 31) >> 5) | 1;  // words per membership row, odd: no bank conflicts
  uint32_t* bits = psm;                                                                // [rows][nW]
  uint8_t* ov = reinterpret_cast<uint8_t*>(bits + static_cast<size_t>(kPairSegment) * nW);  // [rows][32]
  for (int x = tid; x < rows * nW; x += 256) bits[x] = 0u;
  __syncthreads();
  const int32_t* cb = crit + (static_cast<size_t>(bh) * nB + lo) * k_c;
  const int total = rows * k_c;
  for (int x0 = tid; x0 < total; x0 += 256 * 16) {  // 16 loads in flight per thread
    int jv[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) jv[u] = (x0 + 256 * u < total) ? __ldg(cb + x0 + 256 * u) : -1;
#pragma unroll
    for (int u = 0; u < 16; ++u)
      if (jv[u] >= 0) atomicOr(&bits[((x0 + 256 * u) / k_c) * nW + (jv[u] >> 5)], 1u << (jv[u] & 31));
  }
  __syncthreads();
  // ov[r][d-1] = |crit(lo+r) ^ crit(lo+r+d)| for d = 1..32 inside the segment (0 past it)
  for (int x = tid; x < rows * kPairWindow; x += 256) {
    const int r = x / kPairWindow, r2 = r + 1 + x % kPairWindow;
    int v = 0;
    if (r2 < rows)
      for (int w = 0; w < nW; ++w) v += __popc(bits[r * nW + w] & bits[r2 * nW + w]);
    ov[x] = static_cast<uint8_t>(min(v, 254));
  }
  __syncthreads();
  if (tid < 32) {
    int2* out = pairs + static_cast<size_t>(bh) * nB + lo;
    unsigned long long used = 0ull;  // bit k: row r + k already in a tile (warp-uniform)
    int np = 0;
    unsigned nxt = ov[lane];
    for (int r = 0; r < rows; ++r) {
      const unsigned cur = nxt;
      if (r + 1 < rows) nxt = ov[(r + 1) * kPairWindow + lane];
      if (used & 1ull) {
        used >>= 1;
        continue;
      }
      const bool ok = r + 1 + lane < rows && !((used >> (1 + lane)) & 1ull);
      const unsigned key = ok ? ((cur + 1u) << 5) | (31u - static_cast<unsigned>(lane)) : 0u;
      const unsigned best = __reduce_max_sync(0xffffffffu, key);
      const int d = best ? 1 + (31 - static_cast<int>(best & 31u)) : 0;
      if (lane == 0) out[np] = make_int2(lo + r, d ? lo + r + d : -1);
      ++np;
      if (d) used |= 1ull << d;
      used >>= 1;
    }
    if (lane == 0) counts[static_cast<size_t>(bh) * gridDim.x + seg] = np;
  }
}

// ---- whole-head pairing (whole_head_pairing(g)). Pairing is free to choose any partner: a
// row's result depends only on its own critical blocks. The same greedy as pair_kernel (each
// block in ascending order not yet in a tile takes the free block among the next ones that
// shares the most critical blocks with it, ties to the nearest), but over the whole head
// with a window of 127 blocks instead of 64-block segments and 32: 2.4-4.9 % fewer union
// steps on the 720p heads. The scan is sequential per head, so it is used only where the
// attention it saves outweighs it (long heads).
constexpr int kScanWindow = 127;
constexpr int kWinRows = 32;  // rows per CTA of the window table

// win[bh][r][d-1] = min(|crit(r) & crit(r+d)|, 255) for d = 1..127 (0 past the head's end).
// One CTA per 32 rows: the critical sets of rows r0 .. r0+32+126 as bitsets in shared memory.
__global__ void __launch_bounds__(256) pair_window_kernel(const int32_t* __restrict__ crit, int nB, int k_c,
                                                          uint8_t* __restrict__ win) {
  extern __shared__ uint32_t bsm[];  // [kWinRows + kScanWindow][ld]
  const int bh = blockIdx.y, r0 = kWinRows * blockIdx.x, tid = threadIdx.x;
  const int nW = (nB + 31) >> 5, ld = nW | 1;
  const int nrows = min(kWinRows + kScanWindow, nB - r0);
  for (int x = tid; x < nrows * ld; x += 256) bsm[x] = 0u;
  __syncthreads();
  const int32_t* cb = crit + (static_cast<size_t>(bh) * nB + r0) * k_c;
  for (int x = tid; x < nrows * k_c; x += 256) {
    const int j = __ldg(cb + x);
    atomicOr(&bsm[(x / k_c) * ld + (j >> 5)], 1u << (j & 31));
  }
  __syncthreads();
  uint8_t* out = win + (static_cast<size_t>(bh) * nB + r0) * (kScanWindow + 1);
  for (int x = tid; x < kWinRows * (kScanWindow + 1); x += 256) {
    const int r = x / (kScanWindow + 1), d = x % (kScanWindow + 1) + 1;  // d = 1..128
    if (r0 + r >= nB) break;
    int v = 0;
    if (d <= kScanWindow && r + d < nrows)
      for (int w = 0; w < nW; ++w) v += __popc(bsm[r * ld + w] & bsm[(r + d) * ld + w]);
    out[static_cast<size_t>(r) * (kScanWindow + 1) + d - 1] = static_cast<uint8_t>(min(v, 255));
  }
}

// One warp per head: the greedy scan over the window table. Lane l weighs the partners
// d = l+1, l+33, l+65, l+97 (d = 128 is never one); the blocks already taken among the next
// 128 are a warp-uniform 128-bit mask (bit d-1: block r+d), shifted by one per row. Tiles
// go to pairs[bh][0 .. n) in increasing first block, n to counts[bh].
__global__ void __launch_bounds__(32) pair_scan_kernel(const uint8_t* __restrict__ win, int nB,
                                                       int2* __restrict__ pairs, int* __restrict__ counts) {
  extern __shared__ uint4 tsm[];  // the head's window table, nB x 128 bytes
  const int bh = blockIdx.x, lane = threadIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(win + static_cast<size_t>(bh) * nB * (kScanWindow + 1));
  for (int x = lane; x < nB * 8; x += 32 * 8) {  // 8 loads in flight per lane
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = x + 32 * u < nB * 8 ? __ldg(src + x + 32 * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (x + 32 * u < nB * 8) tsm[x + 32 * u] = v[u];
  }
  __syncwarp();
  const uint32_t* tab = reinterpret_cast<const uint32_t*>(tsm);
  int2* out = pairs + static_cast<size_t>(bh) * nB;
  unsigned long long m_lo = 0ull, m_hi = 0ull;  // bit k of (m_hi:m_lo): block r+1+k already taken
  bool self_taken = false;                      // block r itself was taken by an earlier row
  int np = 0;
  for (int r = 0; r < nB; ++r) {
    // row r: this lane's bytes 4*lane .. 4*lane+3 are the partners d = 4*lane+1 .. 4*lane+4
    const uint32_t cur = tab[static_cast<size_t>(r) * ((kScanWindow + 1) / 4) + lane];
    if (!self_taken) {
      unsigned key = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int d = 4 * lane + e + 1;  // this lane's bytes of the row
        const int k = d - 1;
        const bool taken = k < 64 ? ((m_lo >> k) & 1ull) : ((m_hi >> (k - 64)) & 1ull);
        if (d <= kScanWindow && r + d < nB && !taken) {
          const unsigned ov = (cur >> (8 * e)) & 0xFFu;
          key = max(key, ((ov + 1u) << 8) | static_cast<unsigned>(255 - d));
        }
      }
      const unsigned best = __reduce_max_sync(0xffffffffu, key);
      const int d = best ? 255 - static_cast<int>(best & 0xFFu) : 0;
      if (lane == 0) out[np] = make_int2(r, d ? r + d : -1);
      ++np;
      if (d) {
        const int k = d - 1;
        if (k < 64) m_lo |= 1ull << k;
        else m_hi |= 1ull << (k - 64);
      }
    }
    // move to row r+1: bit 0 says whether r+1 is taken
    self_taken = m_lo & 1ull;
    m_lo = (m_lo >> 1) | (m_hi << 63);
    m_hi >>= 1;
  }
  if (lane == 0) counts[bh] = np;
}

}  // namespace

cudaError_t launch_attention(const Dims& g, const void* q, float sm_scale, const int8_t* q8,
                             const int8_t* k8, const float* q_scale, const float* k_scale,
                             const void* v, const int32_t* crit, int k_c, int m, void* out, char* ws,
                             cudaStream_t st) {
  const WsLayout L = ws_layout(g);
  CUtensorMap tmQ, tmK, tmV, tmH;
  if (!make_tmap_3d(&tmQ, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kHeadDim, g.Npad, g.BH, 128, 16) ||
      !make_tmap_3d(&tmK, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kHeadDim, g.Npad, g.BH, 128, 64) ||
      !make_tmap_3d(&tmV, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kHeadDim, g.N, g.BH, 64, 64) ||
      !make_tmap_3d(&tmH, ws + L.Hbuf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kHeadDim,
                    static_cast<uint64_t>(g.nB) * kHeadDim, g.BH, 64, 64))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
  if (e != cudaSuccess) return e;
  int2* pairs = reinterpret_cast<int2*>(ws + L.pairs);
  int* pair_counts = reinterpret_cast<int*>(ws + L.pair_counts);
  int n_seg = (g.nB + kPairSegment - 1) / kPairSegment;
  if (n_seg > 128) return cudaErrorInvalidValue;  // attn_kernel's tile lookup: 4 segments per lane
  if (whole_head_pairing(g)) {  // pairs over the whole head, one segment
    n_seg = 1;
    uint8_t* win = reinterpret_cast<uint8_t*>(ws + L.pair_window);
    {
      TraceScope ts_("pair_window_kernel", st);
      const int nW = (g.nB + 31) / 32;
      const int smem = (kWinRows + kScanWindow) * (nW | 1) * 4;
      e = cudaFuncSetAttribute(pair_window_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      pair_window_kernel<<<dim3((g.nB + kWinRows - 1) / kWinRows, g.BH), 256, smem, st>>>(crit, g.nB, k_c, win);
    }
    {
      TraceScope ts_("pair_scan_kernel", st);
      const int smem = g.nB * (kScanWindow + 1);
      e = cudaFuncSetAttribute(pair_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      pair_scan_kernel<<<g.BH, 32, smem, st>>>(win, g.nB, pairs, pair_counts);
    }
  } else {
    const int nW = ((g.nB + 31) >> 5) | 1;
    const int psmem = kPairSegment * nW * 4 + kPairSegment * kPairWindow;
    e = cudaFuncSetAttribute(pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, psmem);
    if (e != cudaSuccess) return e;
    TraceScope ts_("pair_kernel", st);
    pair_kernel<<<dim3(n_seg, g.BH), 256, psmem, st>>>(crit, g.nB, k_c, pairs, pair_counts);
  }
  AttnParams p;
  p.pairs = pairs;
  p.pair_counts = pair_counts;
  p.n_seg = n_seg;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.crit = crit;
  p.q = m > 0 ? static_cast<const __nv_bfloat16*>(q) : nullptr;
  p.Z = reinterpret_cast<const float*>(ws + L.Zbuf);
  p.H = reinterpret_cast<const __nv_bfloat16*>(ws + L.Hbuf);
  p.c_s = sm_scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = reinterpret_cast<int*>(ws + L.status);
  p.N = g.N;
  p.nB = g.nB;
  p.k_c = k_c;
  {
    TraceScope ts_("attn_kernel", st);
    attn_kernel<<<dim3(g.nB, g.BH), kAttnThreads, kAttnSmem, st>>>(tmQ, tmK, tmV, tmH, p);
  }
  return cudaGetLastError();
}

}  // namespace sgs
