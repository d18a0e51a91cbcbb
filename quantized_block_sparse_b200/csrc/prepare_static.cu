// prepare_static.cu - sagesla_prepare without a caller-provided workspace.
//
// Some callers cannot call cudaMalloc at the point where they run prepare: code that is
// driven from inside an engine that owns all device memory up front (a fixed arena, a
// plugin host, an inference server with a pre-planned memory budget), or code that must
// not allocate once a latency-critical loop has started, because cudaMalloc can
// synchronize the device and its cost is unbounded. For them this entry point keeps the
// only scratch prepare needs - the per-block channel sums of K for the smoothing mean and
// the device status word - in a file-scope __device__ array of fixed size, so the call
// needs nothing but its inputs and outputs.
//
// Properties callers must know:
//   * The array (kStaticScratchBytes, 24 MiB + 256 B) is part of this library's module:
//     every GPU that loads the library holds it until the process exits.
//   * Shapes whose scratch (B*H*ceil(N/64)*128*4 bytes + 256) exceeds it are rejected with
//     SAGESLA_ERR_UNSUPPORTED before anything is launched.
//   * Host code cannot use the array's name as a device address: the first call on each
//     device (with that device current) looks the address up with cudaGetSymbolAddress
//     and caches it. That first call should therefore come before any stream capture.
//   * All calls share the one array and it keeps the last call's contents; the status
//     word is cleared (cudaMemsetAsync, no allocation) at the start of every call. Calls
//     whose kernels overlap on the GPU (different streams, no ordering between them) race
//     on the array and give wrong results: order them on one stream.
//   * A bounded device wait that gives up is recorded in the array's status word; read it
//     with sagesla_static_scratch_status (which synchronizes the stream). The outputs of
//     such a call are invalid.
#include <mutex>

#include "../../include/sagesla.h"
#include "sagesla_internal.h"

namespace sgs {
namespace {

constexpr size_t kStaticScratchBytes = (24u << 20) + 256u;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_prepare_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of the static scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_prepare_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace sgs

extern "C" int sagesla_prepare_static_scratch(const sagesla_shape* shape, const void* q,
                                              const void* k, const void* v, float sm_scale,
                                              int8_t* q8, int8_t* k8, float* q_scale,
                                              float* k_scale, float* k_mean, float* q_bar,
                                              float* k_bar, void* h, float* z, void* stream) {
  if (!shape) return SAGESLA_ERR_INVALID_ARG;
  if (shape->B < 1 || shape->H < 1 || shape->N < 1) return SAGESLA_ERR_INVALID_ARG;
  if (shape->d != sgs::kHeadDim) return SAGESLA_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, q8, k8, q_scale, k_scale, k_mean, q_bar, k_bar, h, z};
  for (const void* p : ptrs)
    if (!sgs::aligned16(p)) return SAGESLA_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !(sm_scale < 3.0e38f)) return SAGESLA_ERR_INVALID_ARG;
  const long long nB = (static_cast<long long>(shape->N) + sgs::kBlock - 1) / sgs::kBlock;
  const long long BH = static_cast<long long>(shape->B) * shape->H;
  if (BH > 65535 || nB > 8192) return SAGESLA_ERR_UNSUPPORTED;
  sgs::Dims g;
  g.B = shape->B;
  g.H = shape->H;
  g.N = shape->N;
  g.BH = static_cast<int>(BH);
  g.nB = static_cast<int>(nB);
  g.Npad = g.nB * sgs::kBlock;
  g.nBp = ((g.nB + 63) / 64) * 64;
  const sgs::WsLayout L = sgs::ws_layout(g);
  // prepare touches only the status word and the partial sums, which come first.
  const size_t need = L.mu_part + static_cast<size_t>(g.BH) * g.nB * sgs::kHeadDim * 4;
  if (need > sgs::kStaticScratchBytes) return SAGESLA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (sgs::scratch_address(&scratch) != cudaSuccess) return SAGESLA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(static_cast<char*>(scratch) + L.status, 0, 256, st) != cudaSuccess)
    return SAGESLA_ERR_CUDA;
  const cudaError_t e = sgs::launch_prepare(g, q, k, v, sm_scale, q8, k8, q_scale, k_scale,
                                            k_mean, q_bar, k_bar, h, z,
                                            static_cast<char*>(scratch), st);
  return e == cudaSuccess ? SAGESLA_OK : SAGESLA_ERR_CUDA;
}

extern "C" int sagesla_static_scratch_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SAGESLA_ERR_CUDA;
  void* scratch = nullptr;
  if (sgs::scratch_address(&scratch) != cudaSuccess) return SAGESLA_ERR_CUDA;
  int word = 0;  // the status word sits at offset 0 of the array (workspace layout)
  if (cudaMemcpy(&word, scratch, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SAGESLA_ERR_CUDA;
  if (word & sgs::kStatusTimeoutBit) return SAGESLA_ERR_TIMEOUT;
  return word ? SAGESLA_ERR_CUDA : SAGESLA_OK;
}
