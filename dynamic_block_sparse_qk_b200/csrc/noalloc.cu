// crisp_route_noalloc: the routing stage for callers that cannot allocate
// device memory.
//
// Some callers of this library are not allowed to call cudaMalloc at all:
// a host framework may reserve the whole device memory up front for its own
// pool and load this library as a plug-in without handing it a workspace, or
// a latency-critical serving loop may not accept the device-wide
// synchronisation that cudaMalloc can cause. For them this entry point runs
// the same routing kernels as crisp_route, with their scratch memory in a
// fixed array that lives in the library's device image instead of a
// caller-provided workspace.
//
// Costs and rules of that choice:
//  * every GPU that loads the library holds CRISP_NOALLOC_SCRATCH_BYTES of
//    device memory for this array until the process exits;
//  * all calls on a device share the one array and it keeps the previous
//    call's contents, so two calls whose kernels overlap on the GPU (for
//    example on two streams without an ordering between them) race and give
//    wrong results — order them on one stream;
//  * problems whose routing scratch exceeds the array are rejected with
//    CRISP_ERR_WORKSPACE before anything is launched;
//  * each call outside stream capture looks up the array's device address
//    (cudaGetSymbolAddress, with the device current); during capture the
//    address of the last lookup on that device is used, so make the first
//    call on a device before any stream capture;
//  * kernel-side errors (a bounded wait that ran out, an out-of-range
//    sequence length) land in a status word at the start of the array:
//    crisp_get_device_status(NULL, ...) reads and clears it.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

using namespace crisp;

namespace {

// Routing scratch for crisp_route_noalloc. In host code this name is only a
// host-side stand-in for the array; the device address comes from
// cudaGetSymbolAddress below and is what the kernels receive.
static __device__ __align__(256) unsigned char g_route_scratch[CRISP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

// Device address of g_route_scratch on the current device. Outside stream
// capture it is looked up on every call (a context that was reset and created
// again may have loaded the module at another address); during capture, when
// no lookup may run, the address cached by the last lookup on this device is
// used, so the first call on a device must come before any capture.
int crisp::noalloc_scratch(void** out, cudaStream_t st) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CRISP_ERR_CUDA;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return CRISP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_route_scratch) != cudaSuccess || !addr) return CRISP_ERR_CUDA;
    g_scratch_addr[dev] = addr;
  }
  if (!g_scratch_addr[dev]) return CRISP_ERR_CUDA;
  *out = g_scratch_addr[dev];
  return CRISP_OK;
}


extern "C" int crisp_route_noalloc(const crisp_params* p, const void* q, const void* k,
                                   int32_t* pattern, float* score, float* p_v, float* p_s,
                                   void* stream) {
  const int s = crisp_check_params(p);
  if (s != CRISP_OK) return s;
  if (!q || !k || !pattern || !score || !p_v || !p_s) return CRISP_ERR_ARG;
  auto al = [](const void* ptr, size_t a) { return reinterpret_cast<uintptr_t>(ptr) % a == 0; };
  if (!al(q, 16) || !al(k, 16) || !al(pattern, 4) || !al(score, 4) || !al(p_v, 4) || !al(p_s, 4))
    return CRISP_ERR_ARG;
  // The routing kernels use only the part of the workspace layout that comes
  // before the pooled-query region.
  const size_t need = make_workspace(*p).qbar;
  if (need > size_t(CRISP_NOALLOC_SCRATCH_BYTES)) return CRISP_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  const int a = noalloc_scratch(&scratch, st);
  if (a != CRISP_OK) return a;
  // The status word and the per-head completion counters must start at zero;
  // every other scratch byte the routing kernels read is written earlier in
  // the same call.
  cudaError_t e = cudaMemsetAsync(scratch, 0, route_clear_bytes(*p), st);
  if (e == cudaSuccess) e = run_route(*p, q, k, scratch, pattern, score, p_v, p_s, st);
  return e == cudaSuccess ? CRISP_OK : CRISP_ERR_CUDA;
}
