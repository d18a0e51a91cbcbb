/*
 * sagesla.h - SageSLA attention forward for NVIDIA B200 (sm_100a), C ABI.
 *
 * SageSLA stacks two attention accelerations described in "TurboDiffusion Demystified:
 * How It Achieves 100x Faster Video Generation":
 *   - section "Pillar One: Low-Bit Attention Acceleration - SageAttention": Q K^T in
 *     INT8 on tensor cores, with K smoothed against outliers;
 *   - section "Pillar Two: Sparse-Linear Attention - SLA": per query block only the
 *     most important key blocks get exact attention (--sla_topk 0.1 keeps 10%, section
 *     "Hands-On Tutorial"), a light linear-attention term covers the middle, the rest is
 *     skipped.
 *
 * Per (batch, head), with 64-token blocks and head dim d = 128:
 *   (1) mu = per-channel mean of K over the N real tokens; K~ = K - mu.
 *   (2) Q~ = Q * sm_scale (sm_scale = fl32(1/sqrt(d)), passed in).
 *   (3) Q~ and K~ quantized per block to symmetric INT8: s = max|x|/127,
 *       x8 = clamp(rint(x/s), -127, 127), round half to even.
 *   (4) logit l_ij = mean(Q~_i) . mean(K~_j) in fp32; per query-block row the top
 *       k_c = ceil(rho*nB) key blocks are critical, the bottom n_neg = floor(nu*nB)
 *       negligible, the rest (m) marginal; equal logits rank the lower index first.
 *   (5) critical blocks: online-softmax attention, scores (q8.k8) * s_q * s_k,
 *       P rounded to bf16 for P.V with fp32 accumulation.
 *   (6) marginal blocks: phi(x) = elu(x)+1, h_j = phi(K~_j)^T V_j, z_j = phi(K~_j)^T 1,
 *       H_i = sum_marg h_j, Z_i = sum_marg z_j, O_l = phi(Q~) H_i / (phi(Q~) . Z_i).
 *   (7) O = O_s + O_l, rounded to bf16.
 *
 * Conventions for every call below.
 *   - All tensor pointers are DEVICE pointers, contiguous, row-major, 16-byte aligned.
 *     The caller owns every buffer; the library allocates, frees and synchronizes
 *     nothing (except sagesla_check_status, which synchronizes the stream).
 *   - nB = ceil(N/64), Npad = 64*nB, nBp = 64*ceil(nB/64) (pitch of the mask rows).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Return value: SAGESLA_OK, or an error code from host-side validation (nothing is
 *     launched), or SAGESLA_ERR_CUDA if a launch failed. Device-side timeouts of bounded
 *     waits are recorded in the workspace status word; read it with
 *     sagesla_check_status.
 *   - Outputs must not alias inputs. Only d = 128 is supported (else UNSUPPORTED).
 *   - Calls are re-entrant across streams if each stream uses its own workspace.
 */
#ifndef SAGESLA_H
#define SAGESLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAGESLA_OK = 0,
  SAGESLA_ERR_INVALID_ARG = 1, /* null pointer, misalignment, bad ratio or size      */
  SAGESLA_ERR_UNSUPPORTED = 2, /* valid but not implemented (d != 128, sizes > max)  */
  SAGESLA_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed               */
  SAGESLA_ERR_TIMEOUT = 4      /* a bounded device wait gave up (see check_status)   */
} sagesla_status;

typedef struct {
  int B; /* batch                       */
  int H; /* heads                       */
  int N; /* tokens per (batch, head)    */
  int d; /* head dim; must be 128       */
} sagesla_shape;

/* Block counts for one query-block row (step 4).
 * k_c = ceil(rho*nB) (>= 1), n_neg = floor(nu*nB) capped at nB-k_c, m = nB-k_c-n_neg;
 * a product within 1e-9 (relative) of an integer counts as that integer.
 * Requires 0 < rho <= 1 and 0 <= nu < 1. Any output pointer may be NULL. */
int sagesla_counts(const sagesla_shape* shape, double rho, double nu,
                   int* nB, int* k_c, int* n_neg, int* m);

/* Bytes of device workspace that prepare and forward need for this shape (the same
 * buffer serves both). It holds the status word, the per-block channel partial sums
 * of step (1), H_i (bf16 [B,H,nB,d,d]), Z_i (fp32 [B,H,nB,d]) and the linear-branch
 * output (bf16 [B,H,N,d]). Returns 0 for an invalid shape. */
size_t sagesla_workspace_bytes(const sagesla_shape* shape);

/* Zero the workspace status word (enqueued on stream). Call once after allocating. */
int sagesla_reset_status(void* workspace, size_t workspace_bytes, void* stream);

/* Steps (1)-(3), the block means of (4) and the linear states of (6).
 * Inputs : q, k, v  bf16 [B,H,N,d]; sm_scale = fl32(1/sqrt(d)) computed by the caller.
 * Outputs: q8, k8      int8 [B,H,Npad,d] (padded rows written as 0)
 *          q_scale, k_scale fp32 [B,H,nB]
 *          k_mean       fp32 [B,H,d]   (mu)
 *          q_bar, k_bar fp32 [B,H,nB,d] (block means of Q~ and K~ over real tokens)
 *          h            bf16 [B,H,nB,d,d]  h_j[c][e] = sum_t phi(K~_t[c]) V_t[e]
 *          z            fp32 [B,H,nB,d]    z_j[c]    = sum_t phi(K~_t[c])
 * INT8 codes, scales, mu and the block means are bit-exact with a fixed summation
 * order (sequential in token order within a block, then over blocks). */
int sagesla_prepare(const sagesla_shape* shape, const void* q, const void* k,
                    const void* v, float sm_scale, int8_t* q8, int8_t* k8,
                    float* q_scale, float* k_scale, float* k_mean, float* q_bar,
                    float* k_bar, void* h, float* z, void* workspace,
                    size_t workspace_bytes, void* stream);

/* sagesla_prepare for callers that cannot allocate device memory when they call it (an
 * engine that owns every buffer from start-up, a plugin host, a loop that must not call
 * cudaMalloc because it can synchronize the device). The paper has no counterpart: this
 * is an interface variant, not a step of the method.
 * Same inputs and outputs as sagesla_prepare, without a workspace: its scratch (the
 * per-block channel sums of K and the status word) lives in a 24 MiB + 256 B __device__
 * array inside the library, held on every GPU that loads the library until exit.
 * Shapes needing more (B*H*ceil(N/64)*512 + 256 bytes) return SAGESLA_ERR_UNSUPPORTED
 * before any launch. The first call on a device looks up the array's address with
 * cudaGetSymbolAddress and should come before any stream capture. All calls share the
 * array: calls whose kernels overlap on the GPU race on it (order them on one stream).
 * Nothing is allocated. A timed-out device wait is recorded in the array's status word:
 * read it with sagesla_static_scratch_status. */
int sagesla_prepare_static_scratch(const sagesla_shape* shape, const void* q, const void* k,
                                   const void* v, float sm_scale, int8_t* q8, int8_t* k8,
                                   float* q_scale, float* k_scale, float* k_mean, float* q_bar,
                                   float* k_bar, void* h, float* z, void* stream);

/* The status word of sagesla_prepare_static_scratch's internal array, for the current
 * device: synchronizes `stream`, then returns SAGESLA_OK, SAGESLA_ERR_TIMEOUT if a bounded
 * device wait of a static-scratch call gave up since that call began (its outputs are
 * invalid), or SAGESLA_ERR_CUDA if the stream reported an error. Each static-scratch call
 * clears the word when it starts. No counterpart in the paper (interface variant). */
int sagesla_static_scratch_status(void* stream);

/* Step (4): block logits, ranking and the per-row block lists.
 * Inputs : q_bar, k_bar fp32 [B,H,nB,d]; rho, nu as in sagesla_counts.
 * Outputs: crit_idx int32 [B,H,nB,k_c]  ascending critical key blocks per row
 *          marg_idx int32 [B,H,nB,m]    ascending marginal key blocks per row (may be
 *                                       NULL when m == 0)
 *          marg_mask bf16 [B,H,nB,nBp]  1.0 where block j is marginal for row i, 0
 *                                       elsewhere (including the pitch padding)
 *          logits   fp32 [B,H,nB,nB]    optional (NULL = not written)
 * Logits use a fixed fp32 order, one fused multiply-add per channel (acc = 0;
 * acc = fl32(qbar[c]*kbar[c] + acc) for c = 0..d-1), so the lists are bit-exact against
 * any implementation that follows it. */
int sagesla_select(const sagesla_shape* shape, const float* q_bar, const float* k_bar,
                   double rho, double nu, int32_t* crit_idx, int32_t* marg_idx,
                   void* marg_mask, float* logits, void* stream);

/* Steps (5)-(7).
 * Inputs : q bf16 [B,H,N,d] (phi(Q~) is recomputed from it), sm_scale, and the
 *          outputs of prepare and select; k_c and m must be the counts of select.
 *          v bf16 [B,H,N,d]. The marginal sums H_i = sum h_j and Z_i = sum z_j are
 *          computed as one GEMM with marg_mask; marg_idx (the same set as a list) is
 *          checked for alignment but not read (it may be NULL when m == 0).
 * Output : out bf16 [B,H,N,d] (rows t >= N are not touched).
 * O_l = phi(Q~) H_i / (phi(Q~) . Z_i) is formed inside the attention kernel and added to
 * O_s in fp32, so the output is rounded to bf16 once.
 * workspace: at least sagesla_workspace_bytes(shape) bytes; forward keeps H, Z, z in
 *          bf16 and the query-block pairing of the attention tiles there. */
int sagesla_forward(const sagesla_shape* shape, const void* q, float sm_scale,
                    const int8_t* q8, const int8_t* k8, const float* q_scale,
                    const float* k_scale, const void* v, const int32_t* crit_idx, int k_c,
                    const void* marg_mask, const int32_t* marg_idx, int m, const void* h,
                    const float* z, void* out, void* workspace, size_t workspace_bytes,
                    void* stream);

/* Step (6), first half, on its own (the GEMM sagesla_forward runs before its attention):
 * H_i = sum of h_j and Z_i = sum of z_j over the marginal key blocks j of query block i
 * ("TurboDiffusion Demystified", section "Pillar Two: Sparse-Linear Attention - SLA": the
 * linear term covers the marginal blocks), as one GEMM with the 0/1 mask.
 * Inputs : marg_mask bf16 [B,H,nB,nBp] and m from sagesla_select; h bf16 [B,H,nB,d,d] and
 *          z fp32 [B,H,nB,d] from sagesla_prepare. 0 <= m <= nB - 1.
 * Outputs: H bf16 [B,H,nB,d,d]: fp32 tensor-core sums of the exact 0/1 x bf16 products,
 *          rounded once (RNE). Z fp32 [B,H,nB,d]: z split into z_hi = bf16(z) and
 *          z_lo = bf16(z - z_hi), each summed in fp32, the two sums added.
 * workspace: at least sagesla_workspace_bytes(shape) bytes (the bf16 split of z and the
 *          status word live there). A row with no marginal block gets H_i = 0, Z_i = 0. */
int sagesla_marginal_sums(const sagesla_shape* shape, const void* marg_mask, int m,
                          const void* h, const float* z, void* H, float* Z, void* workspace,
                          size_t workspace_bytes, void* stream);

/* Synchronize `stream`, then return the workspace status word: SAGESLA_OK, or
 * SAGESLA_ERR_TIMEOUT if a bounded device wait gave up (the affected output is
 * invalid), or SAGESLA_ERR_CUDA if the stream reported an error. */
int sagesla_check_status(const void* workspace, void* stream);

/* ------------------------------------------------------------------------------------
 * Backward pass ("TurboDiffusion Demystified", section "Pillar Two: Sparse-Linear
 * Attention - SLA": the sparse-linear attention is trainable; section "Advanced Guide: How
 * is TurboDiffusion Trained?"). The gradient of steps (1)-(7) for an upstream gradient dO,
 * with the block lists held fixed (they are discrete) and the INT8 quantization read as
 * the identity (straight through): scores Q~.K~^T in full precision, P not rounded. The
 * smoothing mean depends on all of K, so dK sums to zero over tokens.
 * ---------------------------------------------------------------------------------- */

/* Bytes of device workspace sagesla_backward needs (it holds the status word, H, Z, the
 * per-row softmax statistics, dH, dZ, their masked sums and small scratch). */
size_t sagesla_backward_workspace_bytes(const sagesla_shape* shape);

/* dQ, dK, dV (fp32 [B,H,N,d], rows t >= N untouched) for dout bf16 [B,H,N,d].
 * Inputs: q, k, v bf16 [B,H,N,d] and sm_scale as given to the forward; k_mean, h, z from
 * sagesla_prepare; crit_idx, marg_mask (and k_c, m) from sagesla_select (h, z, marg_mask
 * may be NULL when m == 0). Arithmetic: bf16 operands (Q~, K~, V, dO, P, dS, phi, dn) with
 * fp32 accumulation on tensor cores; softmax statistics, D = rowsum(dO o O_s) and the
 * linear-branch denominators in fp32. Deterministic (fixed summation orders, no float
 * atomics). The workspace status word records a timed-out device wait (check_status). */
int sagesla_backward(const sagesla_shape* shape, const void* q, const void* k, const void* v,
                     const void* dout, float sm_scale, const float* k_mean, const void* h,
                     const float* z, const int32_t* crit_idx, int k_c, const void* marg_mask, int m,
                     float* dq, float* dk, float* dv, void* workspace, size_t workspace_bytes,
                     void* stream);

/* ------------------------------------------------------------------------------------
 * W8A8 block-wise INT8 linear layer ("TurboDiffusion Demystified", section "Pillar Three:
 * W8A8 Linear Layer Quantization": weights and activations of the linear layers in INT8,
 * block-wise at 128x128 granularity). Y = X W^T + bias with X [M, K] and W [N, K] each
 * cut into 128x128 tiles (rows x input channels; edge tiles ragged).
 * ---------------------------------------------------------------------------------- */

/* Quantize a bf16 matrix x [rows, K] (row-major) per 128x128 tile: s = fl32(amax/127),
 * x8 = clamp(rint(fl32(x/s)), -127, 127) with ties to even (s = 0 and codes 0 for an
 * all-zero tile). Outputs: x8 int8 [rows, K]; scale fp32 [ceil(rows/128), ceil(K/128)].
 * Serves activations and weights alike. Requires K a multiple of 16 and ceil(rows/128) <=
 * 65535; x and x8 16-byte aligned. The codes and the scales' bits are deterministic. */
int sagesla_w8a8_quantize(const void* x, int rows, int K, int8_t* x8, float* scale,
                          void* stream);

/* Y bf16 [M, N] = sum_kb sx[m/128, kb] * sw[n/128, kb] * (x8[m, kb-tile] . w8[n, kb-tile])
 * + bias[n], from the outputs of sagesla_w8a8_quantize for X (x8, sx) and W (w8, sw).
 * bias: fp32 [N] or NULL. Each K tile's exact integer partial sum is scaled in fp32 (the
 * scale product rounded to fp32) into an fp32 accumulator; the sum is rounded once to
 * bf16. Requires K a multiple of 16 (<= 16384) and N a multiple of 8; x8, w8, y and
 * workspace 16-byte aligned. workspace: >= 256 bytes; its status word records a timed-out
 * device wait (read it with sagesla_check_status). */
int sagesla_w8a8_linear(const int8_t* x8, const float* sx, const int8_t* w8, const float* sw,
                        const float* bias, void* y, int M, int N, int K, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Diagnostics for the failure path (no counterpart in the paper). Launches one small
 * kernel that waits on an mbarrier nothing ever arrives on, through the same bounded wait
 * every kernel of this library uses, with a limit of limit_us microseconds (1..1000000).
 * The wait runs out, the kernel ORs the timeout bit into the workspace status word and
 * returns; the next sagesla_check_status returns SAGESLA_ERR_TIMEOUT and the CUDA context
 * stays usable (clear the word with sagesla_reset_status). workspace: >= 256 bytes, 16-byte
 * aligned. Returns SAGESLA_ERR_INVALID_ARG for a bad pointer or limit, SAGESLA_ERR_CUDA if
 * the launch failed. */
int sagesla_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                  unsigned int limit_us, void* stream);

/* Diagnostics (no counterpart in the paper): the SFU's exponential rate, the denominator
 * of the attention softmax's SFU floor. Launches n_ctas CTAs of 1024 threads, each asking
 * for more than half of an SM's shared memory so that no two share an SM; every thread runs
 * 8 independent chains of `iters` dependent exponentials (x <- 2^-x) in the form `form`:
 * 0 = ex2.approx.ftz.f32 (the form the kernels use), 1 = ex2.approx.f16x2, 2 =
 * ex2.approx.ftz.bf16x2 (forms 1 and 2: two 16-bit exponentials per instruction). CTA b
 * writes three values to out (device memory, caller-owned, out_len >= 3 * n_ctas):
 * out[3b] = exponentials it evaluated, out[3b+1] = SM clock cycles (clock64) around its
 * loop, out[3b+2] = the SM it ran on. exponentials / cycles is the rate per clock of one SM. Asynchronous on `stream`. Returns SAGESLA_ERR_INVALID_ARG
 * for form not 0/1/2, iters outside [1, 2^20], n_ctas outside [1, 1024], a NULL or
 * misaligned out or a short out_len, SAGESLA_ERR_CUDA if the launch failed. */
int sagesla_probe_ex2(int form, int iters, int n_ctas, unsigned long long* out, size_t out_len,
                      void* stream);

/* Launch tracing (diagnostics). While enabled, every kernel launch made by this library
 * is bracketed by a pair of CUDA events recorded on its launch stream. Process-global
 * state, guarded by a mutex; meant for benchmarking, not for concurrent production use. */
int sagesla_trace_enable(int on);

/* Synchronize on the recorded events and write one line per kernel name,
 * "<kernel> <launches> <total_ms>\n", into buf (NUL-terminated, truncated to len); the
 * records are then cleared. Returns SAGESLA_OK, SAGESLA_ERR_CUDA if an event failed, or
 * SAGESLA_ERR_INVALID_ARG if buf was too small. */
int sagesla_trace_read(char* buf, size_t len);

/* Human-readable name of a status code (static string). */
const char* sagesla_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* SAGESLA_H */
