// C ABI of the CRISP library: argument validation and stage dispatch.
// Every entry point validates before launching and returns a crisp_status.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

using namespace crisp;

namespace {

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

int check_params(const crisp_params* p) {
  if (!p) return CRISP_ERR_ARG;
  if (p->batch < 1 || p->h_q < 1 || p->h_kv < 1 || p->seqlen < 1) return CRISP_ERR_SHAPE;
  if (p->h_q % p->h_kv) return CRISP_ERR_SHAPE;
  if (p->head_dim != 64 && p->head_dim != 128) return CRISP_ERR_SHAPE;
  if (p->block != 64 && p->block != 128) return CRISP_ERR_SHAPE;
  const long long nb = (static_cast<long long>(p->seqlen) + p->block - 1) / p->block;
  if (nb < 3 || nb > kMaxBlocks) return CRISP_ERR_SHAPE;
  // the PE softmax partials (ceil(N_b/64) per row) live in a [.][N_b][block] region
  if ((nb + 63) / 64 > p->block) return CRISP_ERR_SHAPE;
  if (static_cast<long long>(p->batch) * p->h_q > 65535) return CRISP_ERR_SHAPE;
  // TMA tile coordinates are 32-bit: every row of q must be addressable
  if (static_cast<long long>(p->batch) * p->h_q * p->seqlen >= (1ll << 31)) return CRISP_ERR_SHAPE;
  if (!(p->alpha > 0.f) || !isfinite(p->alpha)) return CRISP_ERR_ARG;
  if (!(p->gamma > 0.f) || p->gamma > 1.f) return CRISP_ERR_ARG;
  if (!isfinite(p->tau_proxy) || !isfinite(p->tau_jsd)) return CRISP_ERR_ARG;
  if (p->k_min_blocks < 1) return CRISP_ERR_ARG;
  if (p->router != CRISP_ROUTER_CSTRUCT && p->router != CRISP_ROUTER_JSD) return CRISP_ERR_ARG;
  if (p->vs_rule != CRISP_VS_ALPHA && p->vs_rule != CRISP_VS_GAMMA && p->vs_rule != CRISP_VS_ALPHA_MEDIAN)
    return CRISP_ERR_ARG;
  if (!(p->sm_scale >= 0.f) || !isfinite(p->sm_scale)) return CRISP_ERR_ARG;
  if (p->vs_granularity != CRISP_GRAN_TILE && p->vs_granularity != CRISP_GRAN_TOKEN) return CRISP_ERR_ARG;
  if (p->vs_granularity == CRISP_GRAN_TOKEN && p->block != 128) return CRISP_ERR_SHAPE;
  return CRISP_OK;
}

int check_ws(const crisp_params* p, const void* ws, size_t ws_bytes) {
  if (!ws || !aligned(ws, 256)) return CRISP_ERR_ARG;
  if (ws_bytes < make_workspace(*p).total) return CRISP_ERR_WORKSPACE;
  return CRISP_OK;
}

int to_status(cudaError_t e) { return e == cudaSuccess ? CRISP_OK : CRISP_ERR_CUDA; }

}  // namespace



extern "C" {

int crisp_version(void) { return 10200; }

const char* crisp_status_string(int s) {
  switch (s) {
    case CRISP_OK: return "ok";
    case CRISP_ERR_ARG: return "invalid argument";
    case CRISP_ERR_SHAPE: return "unsupported shape";
    case CRISP_ERR_WORKSPACE: return "workspace too small";
    case CRISP_ERR_CUDA: return "CUDA error";
    case CRISP_ERR_TIMEOUT: return "device wait timed out";
    case CRISP_ERR_DEVICE: return "device index out of range";
    default: return "unknown status";
  }
}

int crisp_check_params(const crisp_params* p) { return check_params(p); }

size_t crisp_workspace_size(const crisp_params* p) {
  if (check_params(p) != CRISP_OK) return 0;
  return make_workspace(*p).total;
}

int crisp_route(const crisp_params* p, const void* q, const void* k, void* ws, size_t ws_bytes,
                int32_t* pattern, float* score, float* p_v, float* p_s, void* stream) {
  int s = check_params(p);
  if (s) return s;
  if ((s = check_ws(p, ws, ws_bytes))) return s;
  if (!q || !k || !pattern || !score || !p_v || !p_s) return CRISP_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(pattern, 4) || !aligned(score, 4) ||
      !aligned(p_v, 4) || !aligned(p_s, 4))
    return CRISP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // a prefill starts: clear the status word and the per-head completion counters
  cudaError_t e = cudaMemsetAsync(ws, 0, route_clear_bytes(*p), st);
  if (e == cudaSuccess) e = run_route(*p, q, k, ws, pattern, score, p_v, p_s, st);
  return to_status(e);
}

int crisp_select(const crisp_params* p, const void* q, const void* k, const int32_t* pattern,
                 const float* p_v, const float* p_s, void* ws, size_t ws_bytes, uint8_t* mask,
                 uint8_t* vs_sel, int32_t* tile_idx, int32_t* tile_cnt, void* stream) {
  int s = check_params(p);
  if (s) return s;
  if ((s = check_ws(p, ws, ws_bytes))) return s;
  if (!q || !k || !pattern || !p_v || !p_s || !tile_idx || !tile_cnt) return CRISP_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(pattern, 4) || !aligned(p_v, 4) ||
      !aligned(p_s, 4) || !aligned(tile_idx, 4) || !aligned(tile_cnt, 4))
    return CRISP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = run_select(*p, q, k, pattern, p_v, p_s, ws, mask, tile_idx, tile_cnt, st);
  if (e == cudaSuccess && vs_sel) {
    const Workspace W = make_workspace(*p);
    const size_t bytes = size_t(p->batch) * p->h_q * 2 * n_blocks(*p);
    e = cudaMemcpyAsync(vs_sel, ws_ptr<char>(ws, W.sel), bytes, cudaMemcpyDeviceToDevice, st);
  }
  return to_status(e);
}

int crisp_sparse_prefill(const crisp_params* p, const void* q, const void* k, const void* v,
                         const int32_t* tile_idx, const int32_t* tile_cnt, void* o, float* lse,
                         void* ws, size_t ws_bytes, void* stream) {
  int s = check_params(p);
  if (s) return s;
  if ((s = check_ws(p, ws, ws_bytes))) return s;
  if (!q || !k || !v || !o || !tile_idx || !tile_cnt) return CRISP_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(tile_idx, 4) || !aligned(tile_cnt, 4) || (lse && !aligned(lse, 4)))
    return CRISP_ERR_ARG;
  return to_status(run_attention(*p, q, k, v, tile_idx, tile_cnt, o, lse, ws,
                                 static_cast<cudaStream_t>(stream)));
}

int crisp_dense_prefill(const crisp_params* p, const void* q, const void* k, const void* v,
                        void* o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  int s = check_params(p);
  if (s) return s;
  if ((s = check_ws(p, ws, ws_bytes))) return s;
  if (!q || !k || !v || !o) return CRISP_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      (lse && !aligned(lse, 4)))
    return CRISP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(ws, 0, 8, st);   // a standalone prefill: clear the status word
  if (e == cudaSuccess) e = run_attention(*p, q, k, v, nullptr, nullptr, o, lse, ws, st);
  return to_status(e);
}

int crisp_selftest_pipeline_timeout(const crisp_params* p, const void* q, const void* k, const void* v,
                                    void* o, void* ws, size_t ws_bytes, long long limit_cycles,
                                    void* stream) {
  int s = check_params(p);
  if (s) return s;
  if ((s = check_ws(p, ws, ws_bytes))) return s;
  if (!q || !k || !v || !o) return CRISP_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16)) return CRISP_ERR_ARG;
  if (limit_cycles < 1 || limit_cycles >= (1ll << 20)) return CRISP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the proxy statistics kernel of crisp_route, then the attention kernel of
  // crisp_dense_prefill, both with every pipeline wait cut to limit_cycles
  cudaError_t e = cudaMemsetAsync(ws, 0, route_clear_bytes(*p), st);
  if (e == cudaSuccess) e = run_proxy_stats(*p, q, k, ws, st, limit_cycles);
  if (e == cudaSuccess) e = run_attention(*p, q, k, v, nullptr, nullptr, o, nullptr, ws, st, limit_cycles);
  return to_status(e);
}

int crisp_get_device_status(void* ws, int32_t* status, void* stream) {
  if (!status) return CRISP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!ws) {                 // the scratch array of crisp_route_noalloc on this device
    const int a = noalloc_scratch(&ws, st);
    if (a != CRISP_OK) return a;
  }
  if (!aligned(ws, 256)) return CRISP_ERR_ARG;
  int32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, 8, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return CRISP_ERR_CUDA;
  *status = word;
  return CRISP_OK;
}

}  // extern "C"
