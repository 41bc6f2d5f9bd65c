// crisp_prefill_host: the whole CRISP prefill (route, select, block-sparse
// attention) on inputs and outputs that live in page-locked host memory.
//
// Every KV head with its g query heads is an independent problem (the GQA
// groups share nothing), so the prefill runs chunk by chunk, a chunk being
// one sequence of the batch and kv_per_chunk consecutive KV heads. Two slots
// of device buffers in the caller's workspace alternate between chunks and
// three streams carry the work: the copies in on one, the three stages on the
// caller's stream, the copies out on a third. While chunk i computes, the
// inputs of chunk i+1 cross PCIe one way and the output of chunk i-1 the
// other. Only the rows a sequence holds are copied (one 2-D copy per tensor
// and chunk).
#include <vector>

#include "common.cuh"
#include "kernels.h"

using namespace crisp;

namespace {

struct Slot {
  size_t q, k, v, o, lse, pattern, score, p_v, p_s, tidx, tcnt, ws;
};

struct HostLayout {
  size_t lens;         // int32[batch]            device copy of the lengths
  size_t pattern_log;  // int32[batch * h_q]      routes of every head
  size_t status_log;   // int32[2 * n_chunks]     each chunk's status word
  Slot slot[2];
  size_t slot_ws_bytes;
  size_t total;
};

crisp_params chunk_params(const crisp_params& p, int kv_per_chunk) {
  crisp_params c = p;
  c.batch = 1;
  c.h_kv = kv_per_chunk;
  c.h_q = kv_per_chunk * (p.h_q / p.h_kv);
  c.seq_lens = nullptr;
  return c;
}

HostLayout host_layout(const crisp_params& p, int kv_per_chunk) {
  HostLayout L{};
  const crisp_params c = chunk_params(p, kv_per_chunk);
  const size_t N = size_t(p.seqlen), d = size_t(p.head_dim), nb = size_t(n_blocks(p));
  const size_t cq = size_t(c.h_q), ck = size_t(c.h_kv);
  const size_t chunks = size_t(p.batch) * size_t(p.h_kv / kv_per_chunk);
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  L.lens = take(size_t(p.batch) * 4);
  L.pattern_log = take(size_t(p.batch) * p.h_q * 4);
  L.status_log = take(2 * chunks * 4);
  L.slot_ws_bytes = make_workspace(c).total;
  for (int s = 0; s < 2; ++s) {
    Slot& S = L.slot[s];
    S.q = take(cq * N * d * 2);
    S.k = take(ck * N * d * 2);
    S.v = take(ck * N * d * 2);
    S.o = take(cq * N * d * 2);
    S.lse = take(cq * N * 4);
    S.pattern = take(cq * 4);
    S.score = take(cq * 4);
    S.p_v = take(cq * nb * 4);
    S.p_s = take(cq * nb * 4);
    S.tidx = take(cq * nb * nb * 4);
    S.tcnt = take(cq * nb * 4);
    S.ws = take(L.slot_ws_bytes);
  }
  L.total = off;
  return L;
}

bool page_locked(const void* ptr) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    cudaGetLastError();          // a plain pageable pointer may leave an error behind
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

int check_host_args(const crisp_params* p, int kv_per_chunk) {
  const int s = crisp_check_params(p);
  if (s != CRISP_OK) return s;
  if (p->seq_lens) return CRISP_ERR_ARG;       // lengths come as a host array here
  if (kv_per_chunk < 1 || p->h_kv % kv_per_chunk) return CRISP_ERR_ARG;
  return CRISP_OK;
}

// Streams and events of one call, released on every exit path.
struct Resources {
  cudaStream_t s_in = nullptr, s_out = nullptr;
  std::vector<cudaEvent_t> ev;
  ~Resources() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
  }
  cudaError_t event(cudaEvent_t* e) {
    cudaError_t r = cudaEventCreateWithFlags(e, cudaEventDisableTiming);
    if (r == cudaSuccess) ev.push_back(*e);
    return r;
  }
};

}  // namespace

extern "C" size_t crisp_prefill_host_workspace_size(const crisp_params* p, int kv_per_chunk) {
  if (check_host_args(p, kv_per_chunk) != CRISP_OK) return 0;
  return host_layout(*p, kv_per_chunk).total;
}

extern "C" int crisp_prefill_host(const crisp_params* p, const void* q, const void* k, const void* v,
                                  void* o, float* lse, const int32_t* seq_lens, int32_t* pattern,
                                  int kv_per_chunk, void* ws, size_t ws_bytes, void* stream) {
  int s = check_host_args(p, kv_per_chunk);
  if (s != CRISP_OK) return s;
  if (!q || !k || !v || !o || !ws) return CRISP_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % 256) return CRISP_ERR_ARG;
  const HostLayout L = host_layout(*p, kv_per_chunk);
  if (ws_bytes < L.total) return CRISP_ERR_WORKSPACE;
  if (!page_locked(q) || !page_locked(k) || !page_locked(v) || !page_locked(o) || (lse && !page_locked(lse)))
    return CRISP_ERR_ARG;
  const int B = p->batch, N = p->seqlen, d = p->head_dim;
  const int g = p->h_q / p->h_kv, ck = kv_per_chunk, cq = ck * g;
  std::vector<int32_t> lens(size_t(B), N);
  if (seq_lens) {
    for (int b = 0; b < B; ++b) {
      if (seq_lens[b] <= 2 * p->block || seq_lens[b] > N) return CRISP_ERR_SHAPE;
      lens[size_t(b)] = seq_lens[b];
    }
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(ws);
  Resources R;
  cudaEvent_t start, ev_in[2], ev_cmp[2], ev_out[2];
  cudaError_t e = cudaStreamCreateWithFlags(&R.s_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&R.s_out, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = R.event(&start);
  for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
    e = R.event(&ev_in[i]);
    if (e == cudaSuccess) e = R.event(&ev_cmp[i]);
    if (e == cudaSuccess) e = R.event(&ev_out[i]);
  }
  if (e != cudaSuccess) return CRISP_ERR_CUDA;
  int32_t* lens_dev = reinterpret_cast<int32_t*>(base + L.lens);
  int32_t* pattern_log = reinterpret_cast<int32_t*>(base + L.pattern_log);
  int32_t* status_log = reinterpret_cast<int32_t*>(base + L.status_log);
  const size_t chunks = size_t(B) * size_t(p->h_kv / ck);

  // the pipeline starts after the work already queued on the caller's stream
  e = cudaMemcpyAsync(lens_dev, lens.data(), size_t(B) * 4, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(status_log, 0, 2 * chunks * 4, st);
  if (e == cudaSuccess) e = cudaEventRecord(start, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(R.s_in, start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(R.s_out, start, 0);

  const size_t row = size_t(d) * 2;                       // bytes of one q / k / v / o row
  const size_t head = size_t(N) * row;                     // bytes of one head
  bool used[2] = {false, false};
  int status = CRISP_OK;
  size_t ci = 0;
  for (int b = 0; b < B && e == cudaSuccess && status == CRISP_OK; ++b) {
    const int nv = lens[size_t(b)];
    crisp_params pc = chunk_params(*p, ck);
    pc.seq_lens = seq_lens ? lens_dev + b : nullptr;
    for (int h0 = 0; h0 < p->h_kv && e == cudaSuccess && status == CRISP_OK; h0 += ck, ++ci) {
      const int si = int(ci % 2);
      const Slot& S = L.slot[si];
      char* sq = base + S.q;
      char* sk = base + S.k;
      char* sv = base + S.v;
      char* so = base + S.o;
      float* slse = reinterpret_cast<float*>(base + S.lse);
      void* sws = base + S.ws;
      const char* hq = static_cast<const char*>(q) + (size_t(b) * p->h_q + size_t(h0) * g) * head;
      const char* hk = static_cast<const char*>(k) + (size_t(b) * p->h_kv + h0) * head;
      const char* hv = static_cast<const char*>(v) + (size_t(b) * p->h_kv + h0) * head;
      // copies in: the slot's inputs are free once its previous chunk computed
      if (used[si]) e = cudaStreamWaitEvent(R.s_in, ev_cmp[si], 0);
      if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(sq, head, hq, head, size_t(nv) * row, size_t(cq), cudaMemcpyHostToDevice, R.s_in);
      if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(sk, head, hk, head, size_t(nv) * row, size_t(ck), cudaMemcpyHostToDevice, R.s_in);
      if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(sv, head, hv, head, size_t(nv) * row, size_t(ck), cudaMemcpyHostToDevice, R.s_in);
      // v rows past the sequence inside its last 128-row tile meet exact-zero
      // weights in the PV product: they must be finite, so they are zeroed
      const int pad_end = nv + 127 < N ? ((nv + 127) / 128) * 128 : N;
      if (e == cudaSuccess && pad_end > nv)
        e = cudaMemset2DAsync(sv + size_t(nv) * row, head, 0, size_t(pad_end - nv) * row, size_t(ck), R.s_in);
      if (e == cudaSuccess) e = cudaEventRecord(ev_in[si], R.s_in);
      // compute: after the copies in, and after the slot's previous copy out
      if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev_in[si], 0);
      if (e == cudaSuccess && used[si]) e = cudaStreamWaitEvent(st, ev_out[si], 0);
      if (e != cudaSuccess) break;
      int32_t* spat = reinterpret_cast<int32_t*>(base + S.pattern);
      float* sscore = reinterpret_cast<float*>(base + S.score);
      float* spv = reinterpret_cast<float*>(base + S.p_v);
      float* sps = reinterpret_cast<float*>(base + S.p_s);
      int32_t* stidx = reinterpret_cast<int32_t*>(base + S.tidx);
      int32_t* stcnt = reinterpret_cast<int32_t*>(base + S.tcnt);
      status = crisp_route(&pc, sq, sk, sws, L.slot_ws_bytes, spat, sscore, spv, sps, st);
      if (status == CRISP_OK)
        status = crisp_select(&pc, sq, sk, spat, spv, sps, sws, L.slot_ws_bytes, nullptr, nullptr, stidx, stcnt, st);
      if (status == CRISP_OK)
        status = crisp_sparse_prefill(&pc, sq, sk, sv, stidx, stcnt, so, lse ? slse : nullptr, sws,
                                      L.slot_ws_bytes, st);
      if (status != CRISP_OK) break;
      // keep this chunk's routes and status word (the next route on this slot clears it)
      e = cudaMemcpyAsync(pattern_log + size_t(b) * p->h_q + size_t(h0) * g, spat, size_t(cq) * 4,
                          cudaMemcpyDeviceToDevice, st);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(status_log + 2 * ci, sws, 8, cudaMemcpyDeviceToDevice, st);
      if (e == cudaSuccess) e = cudaEventRecord(ev_cmp[si], st);
      // copies out: this sequence's rows of o (and lse)
      if (e == cudaSuccess) e = cudaStreamWaitEvent(R.s_out, ev_cmp[si], 0);
      char* ho = static_cast<char*>(o) + (size_t(b) * p->h_q + size_t(h0) * g) * head;
      if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(ho, head, so, head, size_t(nv) * row, size_t(cq), cudaMemcpyDeviceToHost, R.s_out);
      if (e == cudaSuccess && lse) {
        float* hl = lse + (size_t(b) * p->h_q + size_t(h0) * g) * size_t(N);
        e = cudaMemcpy2DAsync(hl, size_t(N) * 4, slse, size_t(N) * 4, size_t(nv) * 4, size_t(cq),
                              cudaMemcpyDeviceToHost, R.s_out);
      }
      if (e == cudaSuccess) e = cudaEventRecord(ev_out[si], R.s_out);
      used[si] = true;
    }
  }
  // the call returns once every copy and kernel it issued has finished
  const cudaError_t e1 = cudaStreamSynchronize(R.s_in);
  const cudaError_t e2 = cudaStreamSynchronize(R.s_out);
  const cudaError_t e3 = cudaStreamSynchronize(st);
  if (status != CRISP_OK) return status;
  if (e != cudaSuccess || e1 != cudaSuccess || e2 != cudaSuccess || e3 != cudaSuccess) return CRISP_ERR_CUDA;
  // kernel-side errors of any chunk, then the routes
  std::vector<int32_t> log(2 * chunks);
  if (cudaMemcpy(log.data(), status_log, log.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return CRISP_ERR_CUDA;
  if (pattern && cudaMemcpy(pattern, pattern_log, size_t(B) * p->h_q * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return CRISP_ERR_CUDA;
  for (size_t i = 0; i < chunks; ++i)
    if (log[2 * i] != CRISP_OK) return log[2 * i];
  return CRISP_OK;
}
