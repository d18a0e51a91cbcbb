// api.cu - the C ABI of libsagesla: argument validation, workspace layout, TMA tensor-map
// encoding and kernel launches. See include/sagesla.h for the contract of each call.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "../../include/sagesla.h"
#include "sagesla_internal.h"

namespace sgs {

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

WsLayout ws_layout(const Dims& g) {
  WsLayout L;
  size_t off = 0;
  L.status = off;
  off = align256(off + 256);
  L.mu_part = off;
  off = align256(off + static_cast<size_t>(g.BH) * g.nB * kHeadDim * 4);
  L.Hbuf = off;
  off = align256(off + static_cast<size_t>(g.BH) * g.nB * kHeadDim * kHeadDim * 2);
  L.Zbuf = off;
  off = align256(off + static_cast<size_t>(g.BH) * g.nB * kHeadDim * 4);
  L.Zb = off;
  off = align256(off + static_cast<size_t>(g.BH) * g.nB * kHeadDim * 2 * 2);
  L.pairs = off;
  off = align256(off + static_cast<size_t>(g.BH) * g.nB * 8);
  L.pair_counts = off;
  off = align256(off + static_cast<size_t>(g.BH) * ((g.nB + 63) / 64) * 4);
  const bool whole = whole_head_pairing(g);
  L.pair_window = off;
  off = align256(off + (whole ? static_cast<size_t>(g.BH) * g.nB * 128 : 0));
  L.total = off;
  return L;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once (thread-safe static initialisation); nullptr if the driver lacks it.
static EncodeTiledFn get_encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return nullptr;
  }();
  return fn;
}

// 3-D tiled map over a row-major [d2][d1][d0] array; box = box0 x box1 x 1, 128-byte
// swizzle, out-of-range elements read as zero.
bool make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                  uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box0, uint32_t box1) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * elem_bytes, d0 * d1 * elem_bytes};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  memset(map, 0, sizeof(*map));
  return fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ launch tracing
namespace {
struct TraceRec {
  const char* name;
  cudaEvent_t a, b;
};
std::mutex g_trace_mu;
bool g_trace_on = false;
std::vector<TraceRec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t pool_get() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

TraceScope::TraceScope(const char* name, cudaStream_t st) : slot(-1), stream(st) {
  std::lock_guard<std::mutex> lk(g_trace_mu);
  if (!g_trace_on) return;
  TraceRec r{name, pool_get(), pool_get()};
  if (!r.a || !r.b) return;
  cudaEventRecord(r.a, st);
  slot = static_cast<int>(g_recs.size());
  g_recs.push_back(r);
}

TraceScope::~TraceScope() {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  cudaEventRecord(g_recs[slot].b, stream);
}

}  // namespace sgs

using sgs::Dims;

namespace {

constexpr int kMaxBlocks = 8192;  // select sorts up to 8192 keys per row

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int make_dims(const sagesla_shape* s, Dims* g) {
  if (!s) return SAGESLA_ERR_INVALID_ARG;
  if (s->B < 1 || s->H < 1 || s->N < 1 || s->d < 1) return SAGESLA_ERR_INVALID_ARG;
  if (s->d != sgs::kHeadDim) return SAGESLA_ERR_UNSUPPORTED;
  const long long nB = (static_cast<long long>(s->N) + sgs::kBlock - 1) / sgs::kBlock;
  if (nB > kMaxBlocks) return SAGESLA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(s->B) * s->H;
  if (BH > 65535) return SAGESLA_ERR_UNSUPPORTED;  // grid.y / grid.z limit
  g->B = s->B;
  g->H = s->H;
  g->N = s->N;
  g->BH = static_cast<int>(BH);
  g->nB = static_cast<int>(nB);
  g->Npad = g->nB * sgs::kBlock;
  g->nBp = ((g->nB + 63) / 64) * 64;
  return SAGESLA_OK;
}

bool near_integer(double x, long long* r) {
  const double rr = nearbyint(x);
  if (fabs(x - rr) <= 1e-9 * fmax(1.0, fabs(x))) {
    *r = static_cast<long long>(rr);
    return true;
  }
  return false;
}

int counts_impl(int nB, double rho, double nu, int* k_c, int* n_neg, int* m) {
  if (!(rho > 0.0 && rho <= 1.0) || !(nu >= 0.0 && nu < 1.0)) return SAGESLA_ERR_INVALID_ARG;
  long long kc, nn;
  const double xr = rho * nB, xn = nu * nB;
  if (!near_integer(xr, &kc)) kc = static_cast<long long>(ceil(xr));
  if (kc < 1) kc = 1;
  if (kc > nB) kc = nB;
  if (!near_integer(xn, &nn)) nn = static_cast<long long>(floor(xn));
  if (nn < 0) nn = 0;
  if (nn > nB - kc) nn = nB - kc;
  *k_c = static_cast<int>(kc);
  *n_neg = static_cast<int>(nn);
  *m = static_cast<int>(nB - kc - nn);
  return SAGESLA_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? SAGESLA_OK : SAGESLA_ERR_CUDA; }

}  // namespace

extern "C" {

int sagesla_counts(const sagesla_shape* shape, double rho, double nu, int* nB, int* k_c,
                   int* n_neg, int* m) {
  Dims g;
  int rc = make_dims(shape, &g);
  if (rc != SAGESLA_OK) return rc;
  int a, b, c;
  rc = counts_impl(g.nB, rho, nu, &a, &b, &c);
  if (rc != SAGESLA_OK) return rc;
  if (nB) *nB = g.nB;
  if (k_c) *k_c = a;
  if (n_neg) *n_neg = b;
  if (m) *m = c;
  return SAGESLA_OK;
}

size_t sagesla_workspace_bytes(const sagesla_shape* shape) {
  Dims g;
  if (make_dims(shape, &g) != SAGESLA_OK) return 0;
  return sgs::ws_layout(g).total;
}

int sagesla_reset_status(void* workspace, size_t workspace_bytes, void* stream) {
  if (!aligned16(workspace) || workspace_bytes < 256) return SAGESLA_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(workspace, 0, 256, static_cast<cudaStream_t>(stream)));
}

int sagesla_prepare(const sagesla_shape* shape, const void* q, const void* k, const void* v,
                    float sm_scale, int8_t* q8, int8_t* k8, float* q_scale, float* k_scale,
                    float* k_mean, float* q_bar, float* k_bar, void* h, float* z,
                    void* workspace, size_t workspace_bytes, void* stream) {
  Dims g;
  int rc = make_dims(shape, &g);
  if (rc != SAGESLA_OK) return rc;
  const void* ptrs[] = {q, k, v, q8, k8, q_scale, k_scale, k_mean, q_bar, k_bar, h, z, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SAGESLA_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !isfinite(sm_scale)) return SAGESLA_ERR_INVALID_ARG;
  if (workspace_bytes < sgs::ws_layout(g).total) return SAGESLA_ERR_INVALID_ARG;
  return from_cuda(sgs::launch_prepare(g, q, k, v, sm_scale, q8, k8, q_scale, k_scale, k_mean,
                                       q_bar, k_bar, h, z, static_cast<char*>(workspace),
                                       static_cast<cudaStream_t>(stream)));
}

int sagesla_select(const sagesla_shape* shape, const float* q_bar, const float* k_bar,
                   double rho, double nu, int32_t* crit_idx, int32_t* marg_idx, void* marg_mask,
                   float* logits, void* stream) {
  Dims g;
  int rc = make_dims(shape, &g);
  if (rc != SAGESLA_OK) return rc;
  int k_c, n_neg, m;
  rc = counts_impl(g.nB, rho, nu, &k_c, &n_neg, &m);
  if (rc != SAGESLA_OK) return rc;
  const void* ptrs[] = {q_bar, k_bar, crit_idx, marg_mask};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SAGESLA_ERR_INVALID_ARG;
  if (m > 0 && !aligned16(marg_idx)) return SAGESLA_ERR_INVALID_ARG;
  if (logits && !aligned16(logits)) return SAGESLA_ERR_INVALID_ARG;
  return from_cuda(sgs::launch_select(g, q_bar, k_bar, k_c, n_neg, m, crit_idx, marg_idx,
                                      marg_mask, logits, static_cast<cudaStream_t>(stream)));
}

int sagesla_forward(const sagesla_shape* shape, const void* q, float sm_scale, const int8_t* q8,
                    const int8_t* k8, const float* q_scale, const float* k_scale, const void* v,
                    const int32_t* crit_idx, int k_c, const void* marg_mask,
                    const int32_t* marg_idx, int m, const void* h, const float* z, void* out,
                    void* workspace, size_t workspace_bytes, void* stream) {
  Dims g;
  int rc = make_dims(shape, &g);
  if (rc != SAGESLA_OK) return rc;
  if (k_c < 1 || k_c > g.nB || m < 0 || m > g.nB - k_c) return SAGESLA_ERR_INVALID_ARG;
  const void* ptrs[] = {q8, k8, q_scale, k_scale, v, crit_idx, out, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SAGESLA_ERR_INVALID_ARG;
  if (m > 0) {
    const void* lp[] = {q, marg_mask, marg_idx, h, z};
    for (const void* p : lp)
      if (!aligned16(p)) return SAGESLA_ERR_INVALID_ARG;
    if (!(sm_scale > 0.f) || !isfinite(sm_scale)) return SAGESLA_ERR_INVALID_ARG;
  }
  if (workspace_bytes < sgs::ws_layout(g).total) return SAGESLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  cudaError_t e = sgs::launch_linear(g, marg_mask, m, h, z, ws, st);
  if (e != cudaSuccess) return SAGESLA_ERR_CUDA;
  return from_cuda(sgs::launch_attention(g, q, sm_scale, q8, k8, q_scale, k_scale, v, crit_idx, k_c, m,
                                         out, ws, st));
}

int sagesla_marginal_sums(const sagesla_shape* shape, const void* marg_mask, int m, const void* h,
                          const float* z, void* H, float* Z, void* workspace, size_t workspace_bytes,
                          void* stream) {
  Dims g;
  int rc = make_dims(shape, &g);
  if (rc != SAGESLA_OK) return rc;
  if (m < 0 || m > g.nB - 1) return SAGESLA_ERR_INVALID_ARG;
  const void* ptrs[] = {marg_mask, h, z, H, Z, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SAGESLA_ERR_INVALID_ARG;
  const sgs::WsLayout L = sgs::ws_layout(g);
  if (workspace_bytes < L.total) return SAGESLA_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  return from_cuda(sgs::launch_mask_gemm(g, marg_mask, h, z, static_cast<__nv_bfloat16*>(H), Z,
                                         reinterpret_cast<__nv_bfloat16*>(ws + L.Zb),
                                         reinterpret_cast<int*>(ws + L.status),
                                         static_cast<cudaStream_t>(stream)));
}

size_t sagesla_backward_workspace_bytes(const sagesla_shape* shape) {
  Dims g;
  if (make_dims(shape, &g) != SAGESLA_OK) return 0;
  return sgs::backward_workspace_bytes(g);
}

int sagesla_backward(const sagesla_shape* shape, const void* q, const void* k, const void* v,
                     const void* dout, float sm_scale, const float* k_mean, const void* h,
                     const float* z, const int32_t* crit_idx, int k_c, const void* marg_mask, int m,
                     float* dq, float* dk, float* dv, void* workspace, size_t workspace_bytes,
                     void* stream) {
  Dims g;
  int rc = make_dims(shape, &g);
  if (rc != SAGESLA_OK) return rc;
  if (k_c < 1 || k_c > g.nB || m < 0 || m > g.nB - k_c) return SAGESLA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, dout, k_mean, crit_idx, dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SAGESLA_ERR_INVALID_ARG;
  if (m > 0) {
    const void* lp[] = {h, z, marg_mask};
    for (const void* p : lp)
      if (!aligned16(p)) return SAGESLA_ERR_INVALID_ARG;
  }
  if (!(sm_scale > 0.f) || !isfinite(sm_scale)) return SAGESLA_ERR_INVALID_ARG;
  if (workspace_bytes < sgs::backward_workspace_bytes(g)) return SAGESLA_ERR_INVALID_ARG;
  return from_cuda(sgs::launch_backward(g, q, k, v, dout, sm_scale, k_mean, h, z, crit_idx, k_c,
                                        marg_mask, m, dq, dk, dv, static_cast<char*>(workspace),
                                        static_cast<cudaStream_t>(stream)));
}

int sagesla_check_status(const void* workspace, void* stream) {
  if (!aligned16(workspace)) return SAGESLA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SAGESLA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SAGESLA_ERR_CUDA;
  if (word & sgs::kStatusTimeoutBit) return SAGESLA_ERR_TIMEOUT;
  return word ? SAGESLA_ERR_CUDA : SAGESLA_OK;
}

int sagesla_trace_enable(int on) {
  std::lock_guard<std::mutex> lk(sgs::g_trace_mu);
  sgs::g_trace_on = on != 0;
  return SAGESLA_OK;
}

int sagesla_trace_read(char* buf, size_t len) {
  std::lock_guard<std::mutex> lk(sgs::g_trace_mu);
  std::vector<std::string> names;
  std::vector<double> total;
  std::vector<int> count;
  int rc = SAGESLA_OK;
  for (auto& r : sgs::g_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
      rc = SAGESLA_ERR_CUDA;
    size_t k = 0;
    while (k < names.size() && names[k] != r.name) ++k;
    if (k == names.size()) {
      names.push_back(r.name);
      total.push_back(0.0);
      count.push_back(0);
    }
    total[k] += ms;
    count[k] += 1;
    sgs::g_pool.push_back(r.a);
    sgs::g_pool.push_back(r.b);
  }
  sgs::g_recs.clear();
  std::string out;
  char line[160];
  for (size_t k = 0; k < names.size(); ++k) {
    snprintf(line, sizeof(line), "%s %d %.6f\n", names[k].c_str(), count[k], total[k]);
    out += line;
  }
  if (buf && len) {
    const size_t n = out.size() < len - 1 ? out.size() : len - 1;
    memcpy(buf, out.data(), n);
    buf[n] = 0;
    if (n < out.size()) rc = SAGESLA_ERR_INVALID_ARG;
  }
  return rc;
}

const char* sagesla_status_string(int status) {
  switch (status) {
    case SAGESLA_OK: return "ok";
    case SAGESLA_ERR_INVALID_ARG: return "invalid argument";
    case SAGESLA_ERR_UNSUPPORTED: return "unsupported shape";
    case SAGESLA_ERR_CUDA: return "CUDA error";
    case SAGESLA_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"
