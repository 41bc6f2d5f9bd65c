// PatSearch (CRISP paper, Algorithm 2) on sm_100a: proxy attention of the
// last query block against all keys, its vertical / slash block scores
// (the scores Algorithm 3 thresholds), C_struct (Eq. 2) and the JSD router of the
// paper's Appendix A (Algorithm 5).
//
// The b x n proxy map is never stored. One tensor-core pass (proxy_sm100.cu)
// computes, for every proxy row r and key tile kb, the tile-local row max m
// and the two partial sums of exp2(s - m) over tile columns c <= r and c > r.
// Those two sums are exactly the parts of the tile that fall into slash
// blocks kb and kb + 1 (the diagonal of entry (r, j) is indexed by
// j + b - 1 - r). Its last CTA per head merges them into each row's max and
// normaliser; the scores pass here turns the tile statistics into p_v and
// p_s without touching Q or K again.
#include "common.cuh"
#include "kernels.h"

namespace crisp {

// p_v[kb] = (1/R) sum_r w(r,kb) (lo+hi);  p_s[kb] = (1/R) sum_r [w(r,kb) lo(kb) + w(r,kb-1) hi(kb-1)]
// with w(r,kb) = exp2(m(r,kb) - m_r) / l_r. One warp per key block. With the
// C_struct router the first warp of the first CTA of a head also routes it
// (Eq. 2: C_struct = p_v[0] + p_v[N_b-1], VS iff >= tau_proxy), recomputing
// p_v[N_b-1] with the same arithmetic as the warp that stores it.
__global__ void proxy_scores_kernel(crisp_params p, void* ws, float* __restrict__ p_v,
                                    float* __restrict__ p_s, int32_t* __restrict__ pattern,
                                    float* __restrict__ score) {
  const Workspace W = make_workspace(p);
  const int R = p.block, nb = n_blocks(p);
  const int bh = blockIdx.y;
  const int nbv = (seq_len(p, bh / p.h_q) + R - 1) / R;   // this sequence's blocks
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = blockIdx.x * (blockDim.x >> 5) + warp;
  const float* sm = ws_ptr<float>(ws, W.stat_m) + size_t(bh) * nb * R;
  const float* slo = ws_ptr<float>(ws, W.stat_lo) + size_t(bh) * nb * R;
  const float* shi = ws_ptr<float>(ws, W.stat_hi) + size_t(bh) * nb * R;
  const float* rm = ws_ptr<float>(ws, W.row_m) + size_t(bh) * R;
  const float* rl = ws_ptr<float>(ws, W.row_l) + size_t(bh) * R;
  auto block_scores = [&](int j, float& sv, float& ss) {
    sv = 0.f;
    ss = 0.f;
    for (int r = lane; r < R; r += 32) {
      const float il = 1.f / rl[r];
      const size_t o = size_t(j) * R + r;
      const float w = fast_exp2(sm[o] - rm[r]) * il;
      sv += w * (slo[o] + shi[o]);
      ss += w * slo[o];
      if (j > 0) {
        const size_t o1 = o - R;
        ss += fast_exp2(sm[o1] - rm[r]) * il * shi[o1];
      }
    }
    sv = warp_sum(sv) / float(R);
    ss = warp_sum(ss) / float(R);
  };
  float sv = 0.f, ss = 0.f;
  if (kb < nbv) {
    block_scores(kb, sv, ss);
    if (lane == 0) {
      p_v[size_t(bh) * nb + kb] = sv;
      p_s[size_t(bh) * nb + kb] = ss;
    }
  } else if (kb < nb && lane == 0) {                 // past the end of a shorter sequence
    p_v[size_t(bh) * nb + kb] = 0.f;
    p_s[size_t(bh) * nb + kb] = 0.f;
  }
  if (p.router != CRISP_ROUTER_JSD && kb == 0) {     // routed by route_kernel after K pooling otherwise
    float sv_last, ss_last;
    block_scores(nbv - 1, sv_last, ss_last);
    if (lane == 0) {
      const float c = sv + sv_last;
      score[bh] = c;
      pattern[bh] = (c >= p.tau_proxy) ? CRISP_PATTERN_VS : CRISP_PATTERN_PE;
    }
  }
}

// ---------------------------------------------------------------------------
// Block-mean pooling (Algorithms 4 and 5): a block of
// one head per CTA step (16-byte loads, rows split across thread groups,
// smem reduce), grid-stride over blocks. One launch covers K and Q: heads
// y < nk are K heads (skipped unless a query head of the group is PE, or
// pattern == NULL), the next nq are Q heads (only PE heads).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ k,
                                                   const __nv_bfloat16* __restrict__ q,
                                                   crisp_params p, const int32_t* pattern, int nk, int nq,
                                                   float* __restrict__ kbar, float* __restrict__ qbar) {
  constexpr int CPR = D / 8;
  constexpr int RPP = 256 / CPR;   // rows per pass
  __shared__ float part[RPP][D];
  const int R = p.block, nb = n_blocks(p);
  const int tid = threadIdx.x, c = tid % CPR, rg = tid / CPR;
  // Grid-stride over the flat (head, block) space: the blocks of the heads
  // that are needed spread over all CTAs; a head nobody needs costs one check
  // per item.
  for (int item = blockIdx.x; item < (nk + nq) * nb; item += gridDim.x) {
    const int hy = item / nb, kb = item % nb;
    const bool is_k = hy < nk;
    const int hh = is_k ? hy : hy - nk;
    if (pattern) {
      bool any = false;
      if (!is_k) {
        any = pattern[hh] == CRISP_PATTERN_PE;
      } else {
        const int g = p.h_q / p.h_kv;
        const int b = hh / p.h_kv, hk = hh % p.h_kv;
        for (int i = 0; i < g; ++i) any |= pattern[b * p.h_q + hk * g + i] == CRISP_PATTERN_PE;
      }
      if (!any) continue;
    }
    const int len = seq_len(p, hh / (is_k ? p.h_kv : p.h_q));
    const int nbv = (len + R - 1) / R;
    const __nv_bfloat16* x = is_k ? k : q;
    float* out = is_k ? kbar : qbar;
    if (kb < nbv) {
      const int rows = min(R, len - kb * R);         // a partial last block averages what it holds
      const __nv_bfloat16* src = x + (size_t(hh) * p.seqlen + size_t(kb) * R) * D;
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int row = rg; row < rows; row += RPP) {
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
        out[(size_t(hh) * nb + kb) * D + dd] = s / float(rows);
      }
      __syncthreads();
    }
  }
}

// ---------------------------------------------------------------------------
// JSD routing (Appendix A, Algorithm 5): the distance between p_v and the
// pooled estimate softmax(scale * mean(Q_hat) . K_bar[kb]). One CTA (256
// threads) per query head. (C_struct routing happens in the scores kernel.)
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
  const int nb = n_blocks(p), R = p.block;
  const int bh = blockIdx.x;
  const int len = seq_len(p, bh / p.h_q);
  const int nbv = (len + R - 1) / R;              // this sequence's blocks
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* pv = p_v + size_t(bh) * nb;
  const float scale = p.sm_scale > 0.f ? p.sm_scale : rsqrtf(float(D));
  const size_t N = size_t(p.seqlen);
  const __nv_bfloat16* qh = q + (size_t(bh) * N + len - R) * D;
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
  for (int kb = warp; kb < nbv; kb += 8) {
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
  for (int kb = tid; kb < nbv; kb += 256) {
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
  for (int kb = tid; kb < nbv; kb += 256) {
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
cudaError_t launch_pool(const crisp_params& p, const void* k, const void* q, int nk, int nq,
                        const int32_t* pattern, float* kbar, float* qbar, cudaStream_t st) {
  if (nk + nq == 0) return cudaSuccess;
  const int nb = n_blocks(p);
  const unsigned grid = unsigned(min((nk + nq) * nb, 4 * 148));
  const auto* kk = static_cast<const __nv_bfloat16*>(k);
  const auto* qq = static_cast<const __nv_bfloat16*>(q);
  if (p.head_dim == 64)
    pool_kernel<64><<<grid, 256, 0, st>>>(kk, qq, p, pattern, nk, nq, kbar, qbar);
  else
    pool_kernel<128><<<grid, 256, 0, st>>>(kk, qq, p, pattern, nk, nq, kbar, qbar);
  return cudaGetLastError();
}

cudaError_t run_route(const crisp_params& p, const void* q, const void* k, void* ws,
                      int32_t* pattern, float* score, float* p_v, float* p_s, cudaStream_t st,
                      long long wait_limit) {
  const Workspace W = make_workspace(p);
  const int nb = n_blocks(p);
  const int BH = p.batch * p.h_q;
  // proxy statistics (+ row merge in the last CTA of each head), block
  // scores (+ C_struct route by the warp that computes p_v[0])
  cudaError_t e = run_proxy_stats(p, q, k, ws, st, wait_limit);
  if (e != cudaSuccess) return e;
  proxy_scores_kernel<<<dim3((nb + 7) / 8, BH), 256, 0, st>>>(p, ws, p_v, p_s, pattern, score);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (p.router != CRISP_ROUTER_JSD) return cudaSuccess;
  e = launch_pool(p, k, q, p.batch * p.h_kv, 0, nullptr, ws_ptr<float>(ws, W.kbar), nullptr, st);
  if (e != cudaSuccess) return e;
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
