// Self-test of the bounded-wait path every pipelined kernel of the library
// relies on: one CTA waits on an mbarrier that nothing arrives on, with a
// caller-given cycle limit. The wait gives up, records CRISP_ERR_TIMEOUT in
// the workspace status word and the kernel returns, leaving the context
// usable. No copy is in flight and no tensor memory is held.
#include "common.cuh"
#include "sm100.cuh"

using namespace crisp;
using namespace crisp::sm100;

namespace {

constexpr int kSelftestWhere = 99;   // the `where` code the self-test reports

__global__ void wait_selftest_kernel(void* ws, long long limit) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t* status = static_cast<int32_t*>(ws);
    mbar_wait(smem_u32(&bar), 0, &abort_flag, status, kSelftestWhere, limit);
  }
}

}  // namespace

extern "C" int crisp_selftest_wait_timeout(void* ws, long long limit_cycles, void* stream) {
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256) return CRISP_ERR_ARG;
  if (limit_cycles <= 0 || limit_cycles > (1ll << 31)) return CRISP_ERR_ARG;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ws, limit_cycles);
  return cudaGetLastError() == cudaSuccess ? CRISP_OK : CRISP_ERR_CUDA;
}
