// Internal launch entry points shared between the translation units of the
// CRISP library (not part of the public C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/crisp.h"

namespace crisp {

// Block means of nk K heads into kbar and nq Q heads into qbar, one launch
// (with a pattern: K heads only where a query head of the group is PE, Q
// heads only where the head is PE).
cudaError_t launch_pool(const crisp_params& p, const void* k, const void* q, int nk, int nq,
                        const int32_t* pattern, float* kbar, float* qbar, cudaStream_t st);

// Cycle limit of every bounded wait inside the pipelined kernels (about a
// second); the timeout self-test passes a much shorter one.
constexpr long long kDefaultWaitLimit = 1ll << 31;

// Proxy tile statistics of the last query block (tcgen05 kernel).
cudaError_t run_proxy_stats(const crisp_params& p, const void* q, const void* k, void* ws, cudaStream_t st,
                            long long wait_limit = kDefaultWaitLimit);

cudaError_t run_route(const crisp_params& p, const void* q, const void* k, void* ws,
                      int32_t* pattern, float* score, float* p_v, float* p_s, cudaStream_t st,
                      long long wait_limit = kDefaultWaitLimit);

cudaError_t run_select(const crisp_params& p, const void* q, const void* k, const int32_t* pattern,
                       const float* p_v, const float* p_s, void* ws, uint8_t* mask,
                       int32_t* tile_idx, int32_t* tile_cnt, cudaStream_t st);

// Block-sparse (tile_idx != NULL) or dense causal attention (tcgen05 kernel).
cudaError_t run_attention(const crisp_params& p, const void* q, const void* k, const void* v,
                          const int32_t* tile_idx, const int32_t* tile_cnt, void* o, float* lse,
                          void* ws, cudaStream_t st, long long wait_limit = kDefaultWaitLimit);

// Device address of crisp_route_noalloc's scratch array on the current device
// (its first bytes hold the status word, as in a workspace). Looked up again
// on every call outside stream capture; during capture the address cached at
// the last lookup on that device is used. Returns a crisp_status.
int noalloc_scratch(void** out, cudaStream_t st);

}  // namespace crisp
