// sagesla_internal.h - launch entry points shared between the kernel files and the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sgs {

constexpr int kBlock = 64;     // tokens per quantization / sparsity block
constexpr int kHeadDim = 128;  // supported head dim
constexpr int kStatusTimeoutBit = 4;  // device status word bit for a timed-out wait

struct Dims {
  int B, H, N;
  int BH;    // B*H
  int nB;    // ceil(N/64)
  int Npad;  // 64*nB
  int nBp;   // mask row pitch: 64*ceil(nB/64)
};

// Workspace carve-up (byte offsets, 256-aligned).
struct WsLayout {
  size_t status;     // int32[64]
  size_t mu_part;    // fp32 [BH, nB, d]   per-block channel sums of K
  size_t Hbuf;       // bf16 [BH, nB, d, d]
  size_t Zbuf;       // fp32 [BH, nB, d]
  size_t Zb;         // bf16 [BH, nB, 2d]     [z_hi | z_lo], z split into two bf16 parts
  size_t pairs;      // int2 [BH, nB]         query-block pairs of the attention tiles
  size_t pair_counts;  // int32 [BH, ceil(nB/64)] tiles per pairing segment
  size_t pair_window;  // uint8 [BH, nB, 128] critical-set overlaps with the next 127 blocks
  size_t total;
};
WsLayout ws_layout(const Dims& g);
// Whole-head pairing of query blocks (one warp scans a head's blocks in order, its window
// table in shared memory) for heads of 769 to 1664 blocks with at most 256 MiB of tables; for
// shorter heads the sequential scan costs more than the union steps it saves, and longer ones
// do not fit. Otherwise pairs are chosen within segments of 64 blocks.
inline bool whole_head_pairing(const Dims& g) {
  return g.nB > 768 && g.nB <= 1664 && static_cast<size_t>(g.BH) * g.nB * 128 <= (static_cast<size_t>(256) << 20);
}

// prepare.cu
cudaError_t launch_prepare(const Dims& g, const void* q, const void* k, const void* v,
                           float sm_scale, int8_t* q8, int8_t* k8, float* q_scale,
                           float* k_scale, float* k_mean, float* q_bar, float* k_bar, void* h,
                           float* z, char* ws, cudaStream_t st);
// select.cu
cudaError_t launch_select(const Dims& g, const float* q_bar, const float* k_bar, int k_c,
                          int n_neg, int m, int32_t* crit, int32_t* marg, void* mask,
                          float* logits, cudaStream_t st);
// linear.cu
// H_i = sum of h_j and Z_i = sum of z_j over the marginal blocks of i, into the workspace
// (nothing when m == 0).
cudaError_t launch_linear(const Dims& g, const void* mask, int m, const void* h, const float* z,
                          char* ws, cudaStream_t st);
cudaError_t launch_mask_gemm(const Dims& g, const void* mask, const void* h, const float* z,
                             __nv_bfloat16* Hout, float* Zout, __nv_bfloat16* zb, int* status,
                             cudaStream_t st);
// attention.cu
// Critical-block attention, plus (m > 0) the linear term from the workspace's H_i, Z_i and
// phi(Q*sm_scale) recomputed from q; out = O_s + O_l in bf16.
cudaError_t launch_attention(const Dims& g, const void* q, float sm_scale, const int8_t* q8,
                             const int8_t* k8, const float* q_scale, const float* k_scale,
                             const void* v, const int32_t* crit, int k_c, int m, void* out, char* ws,
                             cudaStream_t st);

// backward.cu
size_t backward_workspace_bytes(const Dims& g);
cudaError_t launch_backward(const Dims& g, const void* q, const void* k, const void* v,
                            const void* dout, float sm_scale, const float* k_mean, const void* h,
                            const float* z, const int32_t* crit, int k_c, const void* mask, int m,
                            float* dq, float* dk, float* dv, char* ws, cudaStream_t st);

// Opt-in launch tracing (api.cu): while enabled, a CUDA event pair is recorded on the
// launch stream around every kernel launch, so per-kernel device time can be read back.
struct TraceScope {
  TraceScope(const char* name, cudaStream_t st);
  ~TraceScope();
  int slot;
  cudaStream_t stream;
};

// tensor maps (api.cu)
bool make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                  uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box0, uint32_t box1);

}  // namespace sgs
