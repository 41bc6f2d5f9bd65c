// PatSearch (CRISP paper, Algorithm 2) on sm_100a: proxy attention of the
// last query block against all keys, its vertical / slash block scores
// (Algorithm 3 lines 3-5), C_struct (Eq. 2) and the JSD router of the
// paper's Appendix A (Algorithm 5).
//
// The b x n proxy map is never stored. One pass computes, for every proxy
// row r and key tile kb, the tile-local row max m and the two partial sums of
// exp2(s - m) over tile columns c <= r and c > r. Those two sums are exactly
// the parts of the tile that fall into slash blocks kb and kb + 1 (the
// diagonal of entry (r, j) is indexed by j + b - 1 - r). A merge gives each
// row's max and normaliser, and a final pass turns the tile statistics into
// p_v and p_s without touching Q or K again.
#include "common.cuh"
#include "kernels.h"

namespace crisp {

// Row max / normaliser of the proxy map from the chunk partials.
__global__ void proxy_merge_kernel(crisp_params p, void* ws) {
  const Workspace W = make_workspace(p);
  const int R = p.block, nb = p.seqlen / p.block;
  const int nc = (nb + kProxyChunk - 1) / kProxyChunk;
  const int bh = blockIdx.x, r = threadIdx.x;
  if (r >= R) return;
  const float* cmv = ws_ptr<float>(ws, W.chunk_m) + size_t(bh) * nc * R;
  const float* clv = ws_ptr<float>(ws, W.chunk_l) + size_t(bh) * nc * R;
  float m = -INFINITY;
  for (int c = 0; c < nc; ++c) m = fmaxf(m, cmv[size_t(c) * R + r]);
  float l = 0.f;
  for (int c = 0; c < nc; ++c) l += clv[size_t(c) * R + r] * fast_exp2(cmv[size_t(c) * R + r] - m);
  ws_ptr<float>(ws, W.row_m)[size_t(bh) * R + r] = m;
  ws_ptr<float>(ws, W.row_l)[size_t(bh) * R + r] = l;
}

// p_v[kb] = (1/R) sum_r w(r,kb) (lo+hi);  p_s[kb] = (1/R) sum_r [w(r,kb) lo(kb) + w(r,kb-1) hi(kb-1)]
// with w(r,kb) = exp2(m(r,kb) - m_r) / l_r. One warp per key block.
__global__ void proxy_scores_kernel(crisp_params p, void* ws, float* __restrict__ p_v,
                                    float* __restrict__ p_s) {
  const Workspace W = make_workspace(p);
  const int R = p.block, nb = p.seqlen / p.block;
  const int bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = blockIdx.x * (blockDim.x >> 5) + warp;
  if (kb >= nb) return;
  const float* sm = ws_ptr<float>(ws, W.stat_m) + size_t(bh) * nb * R;
  const float* slo = ws_ptr<float>(ws, W.stat_lo) + size_t(bh) * nb * R;
  const float* shi = ws_ptr<float>(ws, W.stat_hi) + size_t(bh) * nb * R;
  const float* rm = ws_ptr<float>(ws, W.row_m) + size_t(bh) * R;
  const float* rl = ws_ptr<float>(ws, W.row_l) + size_t(bh) * R;
  float sv = 0.f, ss = 0.f;
  for (int r = lane; r < R; r += 32) {
    const float il = 1.f / rl[r];
    const size_t o = size_t(kb) * R + r;
    const float w = fast_exp2(sm[o] - rm[r]) * il;
    sv += w * (slo[o] + shi[o]);
    ss += w * slo[o];
    if (kb > 0) {
      const size_t o1 = o - R;
      ss += fast_exp2(sm[o1] - rm[r]) * il * shi[o1];
    }
  }
  sv = warp_sum(sv);
  ss = warp_sum(ss);
  if (lane == 0) {
    p_v[size_t(bh) * nb + kb] = sv / float(R);
    p_s[size_t(bh) * nb + kb] = ss / float(R);
  }
}

// ---------------------------------------------------------------------------
// Block-mean pooling (Algorithm 4 line 3; Algorithm 5 line 3): one CTA per
// (head, block); 16-byte loads, rows split across thread groups, smem reduce.
// mode 0: K heads (skipped unless `need` says a query head of the group is
// PE, or need == NULL); mode 1: Q heads, only PE heads.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ x,
                                                   crisp_params p, const int32_t* pattern,
                                                   int mode, float* __restrict__ out) {
  constexpr int CPR = D / 8;
  constexpr int RPP = 256 / CPR;   // rows per pass
  __shared__ float part[RPP][D];
  const int R = p.block, nb = p.seqlen / p.block;
  const int hh = blockIdx.y, kb = blockIdx.x;
  if (pattern) {
    if (mode == 1) {
      if (pattern[hh] != CRISP_PATTERN_PE) return;
    } else {
      const int g = p.h_q / p.h_kv;
      const int b = hh / p.h_kv, hk = hh % p.h_kv;
      bool any = false;
      for (int i = 0; i < g; ++i) any |= pattern[b * p.h_q + hk * g + i] == CRISP_PATTERN_PE;
      if (!any) return;
    }
  }
  const int tid = threadIdx.x, c = tid % CPR, rg = tid / CPR;
  const __nv_bfloat16* src = x + (size_t(hh) * p.seqlen + size_t(kb) * R) * D;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int row = rg; row < R; row += RPP) {
    const uint4 u = *reinterpret_cast<const uint4*>(src + size_t(row) * D + c * 8);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h2[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[rg][c * 8 + i] = acc[i];
  __syncthreads();
  for (int dd = tid; dd < D; dd += 256) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < RPP; ++i) s += part[i][dd];
    out[(size_t(hh) * nb + kb) * D + dd] = s / float(R);
  }
}

// ---------------------------------------------------------------------------
// Routing: C_struct (Eq. 2, = p_v[0] + p_v[N_b-1]) or the JSD distance
// (Algorithm 5) between p_v and the pooled estimate softmax(scale *
// mean(Q_hat) . K_bar[kb]). One CTA (256 threads) per query head.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) route_kernel(const __nv_bfloat16* __restrict__ q,
                                                    crisp_params p, void* ws,
                                                    const float* __restrict__ p_v,
                                                    int32_t* __restrict__ pattern,
                                                    float* __restrict__ score) {
  extern __shared__ float zs[];   // [nb]
  __shared__ float qm[D];
  __shared__ float red[32];
  const Workspace W = make_workspace(p);
  const int nb = p.seqlen / p.block, R = p.block;
  const int bh = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* pv = p_v + size_t(bh) * nb;
  if (p.router != CRISP_ROUTER_JSD) {
    if (tid == 0) {
      const float c = pv[0] + pv[nb - 1];
      score[bh] = c;
      pattern[bh] = (c >= p.tau_proxy) ? CRISP_PATTERN_VS : CRISP_PATTERN_PE;
    }
    return;
  }
  const float scale = p.sm_scale > 0.f ? p.sm_scale : rsqrtf(float(D));
  const size_t N = size_t(p.seqlen);
  const __nv_bfloat16* qh = q + (size_t(bh) * N + N - R) * D;
  for (int dd = tid; dd < D; dd += 256) {
    float s = 0.f;
    for (int r = 0; r < R; ++r) s += __bfloat162float(qh[size_t(r) * D + dd]);
    qm[dd] = s / float(R);
  }
  __syncthreads();
  const int b = bh / p.h_q, h = bh % p.h_q;
  const int hk = h / (p.h_q / p.h_kv);
  const float* kbar = ws_ptr<float>(ws, W.kbar) + (size_t(b) * p.h_kv + hk) * nb * D;
  float lmax = -INFINITY;
  for (int kb = warp; kb < nb; kb += 8) {
    float s = 0.f;
    for (int dd = lane; dd < D; dd += 32) s += qm[dd] * kbar[size_t(kb) * D + dd];
    s = warp_sum(s) * scale;
    if (lane == 0) zs[kb] = s;
    lmax = fmaxf(lmax, s);
  }
  if (lane == 0) red[warp] = lmax;
  __syncthreads();
  float zmax = -INFINITY;
  for (int i = 0; i < 8; ++i) zmax = fmaxf(zmax, red[i]);
  __syncthreads();
  float lsum = 0.f;
  for (int kb = tid; kb < nb; kb += 256) {
    const float e = expf(zs[kb] - zmax);
    zs[kb] = e;
    lsum += e;
  }
  lsum = warp_sum(lsum);
  if (lane == 0) red[warp] = lsum;
  __syncthreads();
  float zsum = 0.f;
  for (int i = 0; i < 8; ++i) zsum += red[i];
  __syncthreads();
  // KL(a_hat || m) + KL(a_bar || m), natural log, 0 log 0 = 0.
  float kl = 0.f;
  for (int kb = tid; kb < nb; kb += 256) {
    const float ah = pv[kb], ab = zs[kb] / zsum;
    const float m = 0.5f * (ah + ab);
    if (ah > 0.f) kl += ah * logf(ah / m);
    if (ab > 0.f) kl += ab * logf(ab / m);
  }
  kl = warp_sum(kl);
  if (lane == 0) red[warp] = kl;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
    for (int i = 0; i < 8; ++i) s += red[i];
    const float djs = sqrtf(fmaxf(0.5f * s, 0.f));
    score[bh] = djs;
    pattern[bh] = (djs >= p.tau_jsd) ? CRISP_PATTERN_VS : CRISP_PATTERN_PE;
  }
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
cudaError_t launch_pool(const crisp_params& p, const void* x, int heads, const int32_t* pattern,
                        int mode, float* out, cudaStream_t st) {
  const int nb = p.seqlen / p.block;
  dim3 grid(nb, heads);
  if (p.head_dim == 64)
    pool_kernel<64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), p, pattern, mode, out);
  else
    pool_kernel<128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), p, pattern, mode, out);
  return cudaGetLastError();
}

cudaError_t run_route(const crisp_params& p, const void* q, const void* k, void* ws,
                      int32_t* pattern, float* score, float* p_v, float* p_s, cudaStream_t st) {
  const Workspace W = make_workspace(p);
  const int nb = p.seqlen / p.block;
  const int BH = p.batch * p.h_q;
  cudaError_t e = run_proxy_stats(p, q, k, ws, st);
  if (e != cudaSuccess) return e;
  proxy_merge_kernel<<<BH, p.block, 0, st>>>(p, ws);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  proxy_scores_kernel<<<dim3((nb + 7) / 8, BH), 256, 0, st>>>(p, ws, p_v, p_s);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (p.router == CRISP_ROUTER_JSD) {
    e = launch_pool(p, k, p.batch * p.h_kv, nullptr, 0, ws_ptr<float>(ws, W.kbar), st);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = size_t(nb) * 4;
  if (p.head_dim == 64) {
    cudaFuncSetAttribute(route_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    route_kernel<64><<<BH, 256, smem, st>>>(static_cast<const __nv_bfloat16*>(q), p, ws, p_v, pattern, score);
  } else {
    cudaFuncSetAttribute(route_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    route_kernel<128><<<BH, 256, smem, st>>>(static_cast<const __nv_bfloat16*>(q), p, ws, p_v, pattern, score);
  }
  return cudaGetLastError();
}

}  // namespace crisp
