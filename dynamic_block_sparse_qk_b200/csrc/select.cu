// Index selection on sm_100a: the sink-aware VS index (CRISP paper,
// Algorithm 3, Eq. 3-4), the FlexPrefill gamma VS index (Appendix A,
// Algorithm 6), the PE index (Algorithm 4) and the tile lists that feed the
// block-sparse attention kernel.
#include "common.cuh"
#include "kernels.h"

namespace crisp {

// ---------------------------------------------------------------------------
// VS selection, one CTA (1024 threads) per (query head, direction).
// Scores stay in shared memory. ALPHA: Eq. 4 count, clip, top-k (rank based
// only when the count is below k_min); ALPHA_MEDIAN: the same with the median
// floor of Appendix H (rank selection). GAMMA: rank every block, scatter to
// descending order, fp64 prefix sum, first prefix >= gamma, clip.
// Ranks order by value descending, equal values by lower index.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) vs_select_kernel(crisp_params p, const int32_t* pattern,
                                                         const float* __restrict__ p_v,
                                                         const float* __restrict__ p_s, void* ws) {
  extern __shared__ unsigned char sm[];
  const int nbs = n_blocks(p);                               // stride of the per-block arrays
  float* pv = reinterpret_cast<float*>(sm);                 // [nbs]
  float* sorted = pv + nbs;                                  // [nbs] (GAMMA)
  double* scan = reinterpret_cast<double*>(sorted + nbs); // [1024], 8-byte aligned (2*nbs floats)
  __shared__ int cnt_s, kcut_s;
  __shared__ float med_s[2];
  const Workspace W = make_workspace(p);
  const int bh = blockIdx.x, dir = blockIdx.y;
  const float* src = (dir == 0 ? p_v : p_s) + size_t(bh) * nbs;
  uint8_t* sel = ws_ptr<uint8_t>(ws, W.sel) + (size_t(bh) * 2 + dir) * nbs;
  const int tid = threadIdx.x;
  const int nb = (seq_len(p, bh / p.h_q) + p.block - 1) / p.block;   // this sequence's blocks
  for (int j = nb + tid; j < nbs; j += 1024) sel[j] = 0;
  // Fresh state for this head's PE path, which runs after this kernel in
  // stream order: radix-select histograms (half per direction CTA), the cut
  // state and the completion counters of the histogram and tie kernels.
  {
    uint32_t* hc = ws_ptr<uint32_t>(ws, W.hist_cnt) + size_t(bh) * 4096 + dir * 2048;
    double* hs = ws_ptr<double>(ws, W.hist_sum) + size_t(bh) * 4096 + dir * 2048;
    for (int i = tid; i < 2048; i += 1024) { hc[i] = 0u; hs[i] = 0.0; }
    if (dir == 0 && tid == 0) {
      ws_ptr<PeState>(ws, W.pe_state)[bh] = PeState{};
      uint32_t* cnt = ws_ptr<uint32_t>(ws, W.head_cnt) + size_t(bh) * 4;
      cnt[kCntHist] = 0u;
      cnt[kCntEq] = 0u;
    }
  }
  if (pattern[bh] != CRISP_PATTERN_VS) {
    for (int j = tid; j < nb; j += 1024) sel[j] = 0;
    return;
  }
  for (int j = tid; j < nb; j += 1024) pv[j] = src[j];
  if (tid == 0) { cnt_s = 0; kcut_s = nb; }
  __syncthreads();
  // The selection as bitmasks (one bit per block, the always-kept vertical
  // block 0 / slash block N_b-1 included) for the tile builder.
  auto write_bits = [&]() {
    __syncthreads();                                     // this CTA's sel[] stores are visible
    const int nw = (nbs + 31) / 32, lane = tid & 31;
    uint32_t* bits = ws_ptr<uint32_t>(ws, W.sel_bits) + (size_t(bh) * 2 + dir) * nw;
    const int always = dir == 0 ? 0 : nb - 1;
    for (int w = tid >> 5; w < nw; w += 32) {
      const int j = w * 32 + lane;
      const unsigned m = __ballot_sync(0xffffffffu, j < nb && (j == always || sel[j] != 0));
      if (lane == 0) bits[w] = m;
    }
  };
  auto rank_of = [&](int j) {
    const float x = pv[j];
    int rk = 0;
    for (int i = 0; i < nb; ++i) {
      const float y = pv[i];
      rk += (y > x) || (y == x && i < j);
    }
    return rk;
  };
  int k;
  if (p.vs_rule == CRISP_VS_ALPHA || p.vs_rule == CRISP_VS_ALPHA_MEDIAN) {
    float mu;
    if (p.vs_rule == CRISP_VS_ALPHA) {
      float r = (1.0f - pv[0]) - pv[nb - 1];
      r = fmaxf(r, 0.0f);
      mu = r / float(nb - 2);
    } else {
      // Median of the non-retained blocks 1..N_b-2 (Appendix H): the blocks
      // of ascending rank (m-1)/2 and m/2 among the m = N_b-2 middle scores,
      // ranks made distinct by the block index.
      const int m = nb - 2, klo = (m - 1) / 2, khi = m / 2;
      for (int j = 1 + tid; j < nb - 1; j += 1024) {
        const float x = pv[j];
        int rk = 0;
        for (int i = 1; i < nb - 1; ++i) {
          const float y = pv[i];
          rk += (y < x) || (y == x && i < j);
        }
        if (rk == klo) med_s[0] = x;
        if (rk == khi) med_s[1] = x;
      }
      __syncthreads();
      mu = (m & 1) ? med_s[0] : (med_s[0] + med_s[1]) * 0.5f;
    }
    const float thr = p.alpha * mu;
    int c = 0;
    for (int j = tid; j < nb; j += 1024) c += pv[j] > thr;
    c = __reduce_add_sync(0xffffffffu, c);
    if ((tid & 31) == 0) atomicAdd(&cnt_s, c);
    __syncthreads();
    const int cnt = cnt_s;
    k = min(max(cnt, p.k_min_blocks), nb);
    if (k == cnt) {
      for (int j = tid; j < nb; j += 1024) sel[j] = pv[j] > thr;
    } else {
      for (int j = tid; j < nb; j += 1024) sel[j] = rank_of(j) < k;
    }
    write_bits();
    return;
  }
  // GAMMA (Algorithm 6).
  for (int j = tid; j < nb; j += 1024) sorted[rank_of(j)] = pv[j];
  __syncthreads();
  // Block-wide inclusive prefix sum in fp64: thread t owns a contiguous run.
  const int per = (nb + 1023) / 1024;
  const int j0 = tid * per, j1 = min(j0 + per, nb);
  double run = 0.0;
  for (int j = j0; j < j1; ++j) run += double(sorted[j]);
  scan[tid] = run;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const double v = tid >= off ? scan[tid - off] : 0.0;
    __syncthreads();
    scan[tid] += v;
    __syncthreads();
  }
  double acc = tid > 0 ? scan[tid - 1] : 0.0;
  const double g = double(p.gamma);
  for (int j = j0; j < j1; ++j) {
    acc += double(sorted[j]);
    if (acc >= g) { atomicMin(&kcut_s, j + 1); break; }
  }
  __syncthreads();
  k = min(max(kcut_s, p.k_min_blocks), nb);
  for (int j = tid; j < nb; j += 1024) sel[j] = rank_of(j) < k;
  write_bits();
}

// ---------------------------------------------------------------------------
// PE estimate (Algorithm 4): logits of Q_bar K_bar^T for kb <= qb,
// 64x64 tiles (grid-stride over PE heads and tiles), fp32 FMA; written in
// log2 units into abar together
// with per-(row, tile) max / sum partials. Then a row pass normalises and
// divides by N_b (Algorithm 4 normalises by the total, which for N_b causal
// softmax rows is N_b).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) pe_logits_kernel(crisp_params p, const int32_t* pattern,
                                                        void* ws) {
  constexpr int T = 64, KC = 32;
  __shared__ float qs[KC][T + 1];
  __shared__ float kst[KC][T + 1];
  __shared__ float rmax[T][17], rsum[T][17];
  const Workspace W = make_workspace(p);
  const int nb = n_blocks(p);                               // stride
  const int BH = p.batch * p.h_q;
  const int ntq_max = (nb + T - 1) / T, tiles_max = ntq_max * (ntq_max + 1) / 2;
  // Grid-stride over the flat (head, lower-triangle 64x64 tile) space, so the
  // tiles of all PE heads spread over the CTAs even when a head has only a
  // few; a head that is not PE costs one check per item.
  for (int item = blockIdx.x; item < BH * tiles_max; item += gridDim.x) {
    const int bh = item / tiles_max, tt = item % tiles_max;
    if (pattern[bh] != CRISP_PATTERN_PE) continue;
    const int nbv = (seq_len(p, bh / p.h_q) + p.block - 1) / p.block;   // this sequence's blocks
    const int ntq = (nbv + T - 1) / T;
    if (tt >= ntq * (ntq + 1) / 2) continue;
    {
      int tq = int((sqrtf(8.f * float(tt) + 1.f) - 1.f) * 0.5f);
      while ((tq + 1) * (tq + 2) / 2 <= tt) ++tq;
      while (tq * (tq + 1) / 2 > tt) --tq;
      const int tk = tt - tq * (tq + 1) / 2;
      const int b = bh / p.h_q, h = bh % p.h_q, hk = h / (p.h_q / p.h_kv);
      const float* qbar = ws_ptr<float>(ws, W.qbar) + size_t(bh) * nb * D;
      const float* kbar = ws_ptr<float>(ws, W.kbar) + (size_t(b) * p.h_kv + hk) * nb * D;
      float* abar = ws_ptr<float>(ws, W.abar) + size_t(bh) * nb * nb;
      const float sl2 = (p.sm_scale > 0.f ? p.sm_scale : rsqrtf(float(D))) * kLog2e;
      const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;   // 4x4 micro-tile per thread
      float acc[4][4] = {};
      for (int k0 = 0; k0 < D; k0 += KC) {
        for (int i = tid; i < T * KC; i += 256) {
          const int r = i / KC, c = i % KC;
          const int qr = tq * T + r, kr = tk * T + r;
          qs[c][r] = qr < nbv ? qbar[size_t(qr) * D + k0 + c] : 0.f;
          kst[c][r] = kr < nbv ? kbar[size_t(kr) * D + k0 + c] : 0.f;
        }
        __syncthreads();
    #pragma unroll 8
        for (int c = 0; c < KC; ++c) {
          float a[4], bb[4];
    #pragma unroll
          for (int i = 0; i < 4; ++i) { a[i] = qs[c][ty * 4 + i]; bb[i] = kst[c][tx * 4 + i]; }
    #pragma unroll
          for (int i = 0; i < 4; ++i)
    #pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
      }
      // write logits (log2 units) and per-row partial max / sum over this tile
    #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int qb = tq * T + ty * 4 + i;
        float mx = -INFINITY;
    #pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int kb = tk * T + tx * 4 + j;
          const bool ok = qb < nbv && kb <= qb;
          acc[i][j] = ok ? acc[i][j] * sl2 : -INFINITY;
          if (ok) abar[size_t(qb) * nb + kb] = acc[i][j];
          mx = fmaxf(mx, acc[i][j]);
        }
        float s = 0.f;
    #pragma unroll
        for (int j = 0; j < 4; ++j) s += (acc[i][j] == -INFINITY) ? 0.f : exp2f(acc[i][j] - mx);
        rmax[ty * 4 + i][tx] = mx;
        rsum[ty * 4 + i][tx] = s;
      }
      __syncthreads();
      if (tid < T) {
        const int qb = tq * T + tid;
        if (qb < nbv) {
          float mx = -INFINITY;
          for (int j = 0; j < 16; ++j) mx = fmaxf(mx, rmax[tid][j]);
          float s = 0.f;
          for (int j = 0; j < 16; ++j)
            if (rmax[tid][j] != -INFINITY) s += rsum[tid][j] * exp2f(rmax[tid][j] - mx);
          const int ntile = (nb + T - 1) / T;
          // partials reuse the proxy statistic regions (free once routing is done)
          ws_ptr<float>(ws, W.stat_m)[(size_t(bh) * nb + qb) * ntile + tk] = mx;
          ws_ptr<float>(ws, W.stat_lo)[(size_t(bh) * nb + qb) * ntile + tk] = s;
        }
      }
      __syncthreads();                                      // rmax / rsum are reused
    }
  }
}

// One warp per PE row: combine partials, rewrite abar[qb][kb] = softmax / N_b.
__global__ void pe_normalize_kernel(crisp_params p, const int32_t* pattern, void* ws) {
  const Workspace W = make_workspace(p);
  const int nb = n_blocks(p);                               // stride
  const int bh = blockIdx.y;
  if (pattern[bh] != CRISP_PATTERN_PE) return;
  const int nbv = (seq_len(p, bh / p.h_q) + p.block - 1) / p.block;   // this sequence's blocks
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x * (blockDim.x >> 5) + warp;
  if (qb >= nbv) return;
  const int ntile = (nb + 63) / 64;
  const int nt = qb / 64 + 1;
  const float* pm = ws_ptr<float>(ws, W.stat_m) + (size_t(bh) * nb + qb) * ntile;
  const float* ps = ws_ptr<float>(ws, W.stat_lo) + (size_t(bh) * nb + qb) * ntile;
  float mx = -INFINITY;
  for (int t = lane; t < nt; t += 32) mx = fmaxf(mx, pm[t]);
  mx = warp_max(mx);
  float s = 0.f;
  for (int t = lane; t < nt; t += 32) s += ps[t] * exp2f(pm[t] - mx);
  s = warp_sum(s);
  const float inv = 1.0f / (s * float(nbv));               // Algorithm 4: the total is N_b
  float* row = ws_ptr<float>(ws, W.abar) + (size_t(bh) * nb + qb) * nb;
  for (int kb = lane; kb <= qb; kb += 32) row[kb] = exp2f(row[kb] - mx) * inv;
}

// ---------------------------------------------------------------------------
// Gamma cut over the PE triangle by radix select on the float bit patterns
// (positive floats order like their bits). Level 0: bits 31..20, level 1:
// bits 19..8, level 2: bits 7..0. Bucket counts and fp64 sums per head.
// ---------------------------------------------------------------------------
__device__ inline void level_geom(int level, int& shift, int& nbk) {
  shift = level == 0 ? 20 : (level == 1 ? 8 : 0);
  nbk = level == 2 ? 256 : 4096;
}

// The highest bucket whose descending cumulative sum (above_sum + buckets
// above + itself) reaches gamma; run by the 256 threads of the last histogram
// CTA of a head. suf: 257 doubles of shared scratch, ctl: 2 ints.
__device__ void pe_find(const crisp_params& p, PeState* stp, uint32_t* gc, double* gs, int level,
                        double* suf, int* ctl) {
  int shift, nbk;
  level_geom(level, shift, nbk);
  const int tid = threadIdx.x;
  const int per = nbk / 256;   // 16 (levels 0, 1) or 1 (level 2)
  int& best = ctl[0];
  int& lowest = ctl[1];
  // thread t owns buckets counted from the top: nbk-1 - (t*per + i)
  double own = 0.0;
  for (int i = 0; i < per; ++i) own += __ldcg(gs + (nbk - 1 - (tid * per + i)));
  suf[tid] = own;
  if (tid == 0) { best = -1; lowest = 1 << 30; }
  __syncthreads();
  for (int bk = tid; bk < nbk; bk += 256)
    if (__ldcg(gc + bk)) atomicMin(&lowest, bk);
  for (int off = 1; off < 256; off <<= 1) {
    const double v = tid >= off ? suf[tid - off] : 0.0;
    __syncthreads();
    suf[tid] += v;
    __syncthreads();
  }
  const double g = double(p.gamma);
  const double above0 = stp->above_sum;
  double run = above0 + (tid > 0 ? suf[tid - 1] : 0.0);
  int cand = -1;
  double cand_above = 0.0;                 // sum strictly above this thread's candidate bucket
  for (int i = 0; i < per; ++i) {
    const int bk = nbk - 1 - (tid * per + i);
    const double v = __ldcg(gs + bk);
    if (run + v >= g) { cand = bk; cand_above = run; atomicMax(&best, bk); break; }
    run += v;
  }
  __syncthreads();
  // the owner of the chosen bucket (ranges are disjoint: exactly one thread)
  // hands over the sum strictly above it
  double* above_s = suf + 256;
  if (cand >= 0 && cand == best) *above_s = cand_above;
  __syncthreads();
  if (tid == 0) {
    PeState s = *stp;
    int cut = best;
    if (cut < 0 && level > 0 && lowest < nbk) cut = lowest;  // rounding fell short: whole range
    if (cut < 0) {
      s.all = 1;                       // the whole triangle sums below gamma
    } else {
      // every bucket above the lowest non-empty one: the scan total without it
      const double above = cut == best ? *above_s : above0 + suf[255] - __ldcg(gs + cut);
      s.prefix |= uint32_t(cut) << shift;
      s.above_sum = above;
      if (level == 2) {
        const float tv = __uint_as_float(s.prefix);
        const double need = g - above;
        double m = ceil(need / double(tv));
        if (m < 1.0) m = 1.0;
        const double cap = double(__ldcg(gc + cut));
        if (m > cap) m = cap;
        s.m_equal = uint32_t(m);
      }
    }
    *stp = s;
  }
  __syncthreads();
  for (int i = tid; i < nbk; i += 256) { gc[i] = 0; gs[i] = 0.0; }
}

// Adds this lane's entry (bucket bk, value s; take = false: no entry) to a
// shared-memory histogram of counts and fp64 sums. The entries of a row are
// close in value, so the lanes of a warp mostly hit one or two buckets:
// lanes with the same bucket combine first (each lane links to the next lane
// of its bucket, five pointer-jumping steps leave the group's sum in its
// lowest lane) and only that lane updates shared memory. All 32 lanes call.
__device__ inline void hist_add_warp(uint32_t* hc, double* hs, bool take, uint32_t bk, double s) {
  const int lane = threadIdx.x & 31;
  if (!__any_sync(0xffffffffu, take)) return;
  const unsigned peers = __match_any_sync(0xffffffffu, bk);
  const unsigned above = lane == 31 ? 0u : peers & (0xFFFFFFFFu << (lane + 1));
  int nxt = above ? __ffs(above) - 1 : -1;
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int src = nxt >= 0 ? nxt : lane;
    const double o = __shfl_sync(0xffffffffu, s, src);
    const int on = __shfl_sync(0xffffffffu, nxt, src);
    if (nxt >= 0) {
      s += o;
      nxt = on;
    }
  }
  if (take && (peers & ((1u << lane) - 1u)) == 0u) {
    atomicAdd(&hc[bk], uint32_t(__popc(peers)));
    atomicAdd(&hs[bk], s);
  }
}

__global__ void __launch_bounds__(256) pe_hist_kernel(crisp_params p, const int32_t* pattern,
                                                      void* ws, int level) {
  __shared__ uint32_t hc[4096];
  __shared__ double hs[4096];
  const Workspace W = make_workspace(p);
  const int nb = n_blocks(p);                               // stride
  const int bh = blockIdx.y;
  if (pattern[bh] != CRISP_PATTERN_PE) return;
  const PeState st = ws_ptr<PeState>(ws, W.pe_state)[bh];
  if (st.all) return;
  const int nbv = (seq_len(p, bh / p.h_q) + p.block - 1) / p.block;   // this sequence's blocks
  int shift, nbk;
  level_geom(level, shift, nbk);
  for (int i = threadIdx.x; i < nbk; i += 256) { hc[i] = 0; hs[i] = 0.0; }
  __syncthreads();
  const float* abar = ws_ptr<float>(ws, W.abar) + size_t(bh) * nb * nb;
  const int rows_per = 8;
  const int q0 = blockIdx.x * rows_per, q1 = min(q0 + rows_per, nbv);
  const uint32_t hi_shift = shift + (level == 2 ? 8 : 12);
  for (int qb = q0; qb < q1; ++qb) {
    const float* row = abar + size_t(qb) * nb;
    for (int c0 = 0; c0 <= qb; c0 += 256) {          // uniform trip count: the whole CTA iterates
      const int kb = c0 + int(threadIdx.x);
      bool take = false;
      uint32_t bk = 0xFFFFFFFFu;
      double s = 0.0;
      if (kb <= qb) {
        const float v = row[kb];
        const uint32_t u = __float_as_uint(v);
        if (level == 0 || (u >> hi_shift) == (st.prefix >> hi_shift)) {
          take = true;
          bk = (u >> shift) & uint32_t(nbk - 1);
          s = double(v);
        }
      }
      hist_add_warp(hc, hs, take, bk, s);
    }
  }
  __syncthreads();
  uint32_t* gc = ws_ptr<uint32_t>(ws, W.hist_cnt) + size_t(bh) * 4096;
  double* gs = ws_ptr<double>(ws, W.hist_sum) + size_t(bh) * 4096;
  for (int i = threadIdx.x; i < nbk; i += 256)
    if (hc[i]) { atomicAdd(&gc[i], hc[i]); atomicAdd(&gs[i], hs[i]); }
  // The last CTA of this head to finish finds the cut bucket.
  __threadfence();
  __syncthreads();
  int* ctl = reinterpret_cast<int*>(hc);       // the shared histogram is free now
  uint32_t* cnt = ws_ptr<uint32_t>(ws, W.head_cnt) + size_t(bh) * 4 + kCntHist;
  if (threadIdx.x == 0) ctl[0] = atomicAdd(cnt, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!ctl[0]) return;
  __threadfence();
  pe_find(p, ws_ptr<PeState>(ws, W.pe_state) + bh, gc, gs, level, hs, ctl + 1);
  if (threadIdx.x == 0) *cnt = 0u;
}

// Per-row count of entries equal to the cut value; the last CTA of a head
// turns the counts into an exclusive scan, so the tile builder can take the
// first m_equal of them in flat (row-major) order.
__global__ void __launch_bounds__(256) pe_eqcount_kernel(crisp_params p, const int32_t* pattern, void* ws) {
  __shared__ uint32_t part[256];
  __shared__ int last;
  const Workspace W = make_workspace(p);
  const int nbs = n_blocks(p);                              // stride
  const int bh = blockIdx.y;
  if (pattern[bh] != CRISP_PATTERN_PE) return;
  const PeState st = ws_ptr<PeState>(ws, W.pe_state)[bh];
  if (st.all) return;
  const int nb = (seq_len(p, bh / p.h_q) + p.block - 1) / p.block;    // this sequence's blocks
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qb = blockIdx.x * 8 + warp;
  uint32_t* ec = ws_ptr<uint32_t>(ws, W.eq_cnt) + size_t(bh) * nbs;
  if (qb < nb) {
    const float tv = __uint_as_float(st.prefix);
    const float* row = ws_ptr<float>(ws, W.abar) + (size_t(bh) * nbs + qb) * nbs;
    uint32_t c = 0;
    for (int kb = lane; kb <= qb; kb += 32) c += row[kb] == tv;
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) ec[qb] = c;
  }
  __threadfence();
  __syncthreads();
  uint32_t* cnt = ws_ptr<uint32_t>(ws, W.head_cnt) + size_t(bh) * 4 + kCntEq;
  if (tid == 0) last = atomicAdd(cnt, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  const int per = (nb + 255) / 256;
  const int j0 = min(tid * per, nb), j1 = min(j0 + per, nb);
  uint32_t s = 0;
  for (int j = j0; j < j1; ++j) s += __ldcg(ec + j);
  part[tid] = s;
  __syncthreads();
  for (int off = 1; off < 256; off <<= 1) {
    const uint32_t v = tid >= off ? part[tid - off] : 0u;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  uint32_t run = tid > 0 ? part[tid - 1] : 0u;
  for (int j = j0; j < j1; ++j) {
    const uint32_t c = __ldcg(ec + j);
    ec[j] = run;
    run += c;
  }
  if (tid == 0) *cnt = 0u;
}

// ---------------------------------------------------------------------------
// The PE gamma cut of one head in one CTA, for triangles that fit in shared
// memory (N_b(N_b+1)/2 <= kPeSmallMax, i.e. N_b <= 256: sequences up to 32k
// tokens at block 128). It replaces the normalisation, the three histogram
// launches and the tie count of the multi-kernel path with the same
// arithmetic: rows normalised as in pe_normalize_kernel (written back for the
// tile builder and kept in shared memory in flat order), the same three-level
// radix select with fp64 bucket sums and the same cut search, and the same
// per-row tie counts turned into an exclusive scan; it leaves the PeState and
// eq_cnt that build_tiles_kernel reads. One CTA of 1024 threads per head.
// ---------------------------------------------------------------------------
constexpr int kPeSmallMax = 256 * 257 / 2;
constexpr int kPeSmallThreads = 1024;
constexpr size_t kPeSmallSmem = size_t(kPeSmallMax) * 4 + 4096 * 4 + 4096 * 8 + (kPeSmallThreads + 2) * 8 + 256 * 4;

__global__ void __launch_bounds__(kPeSmallThreads) pe_small_cut_kernel(crisp_params p, const int32_t* pattern,
                                                                      void* ws) {
  extern __shared__ __align__(16) unsigned char sm_raw[];
  double* hs = reinterpret_cast<double*>(sm_raw);                       // [4096]
  double* scan = hs + 4096;                                             // [1024 + 2]
  uint32_t* hc = reinterpret_cast<uint32_t*>(scan + kPeSmallThreads + 2);  // [4096]
  uint32_t* rowc = hc + 4096;                                           // [256]
  float* vals = reinterpret_cast<float*>(rowc + 256);                   // [kPeSmallMax]
  __shared__ int ctl[2];
  __shared__ PeState st;
  const Workspace W = make_workspace(p);
  const int nb = n_blocks(p);                               // stride
  const int bh = blockIdx.x;
  if (pattern[bh] != CRISP_PATTERN_PE) return;
  const int nbv = (seq_len(p, bh / p.h_q) + p.block - 1) / p.block;   // this sequence's blocks
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int M = nbv * (nbv + 1) / 2;
  float* abar = ws_ptr<float>(ws, W.abar) + size_t(bh) * nb * nb;
  // (1) rows: combine the logits kernel's (max, sum) partials, normalise,
  // divide by N_b (as pe_normalize_kernel), write back and keep in flat order
  {
    const int ntile = (nb + 63) / 64;
    for (int qb = warp; qb < nbv; qb += kPeSmallThreads / 32) {
      const int nt = qb / 64 + 1;
      const float* pm = ws_ptr<float>(ws, W.stat_m) + (size_t(bh) * nb + qb) * ntile;
      const float* ps = ws_ptr<float>(ws, W.stat_lo) + (size_t(bh) * nb + qb) * ntile;
      float mx = -INFINITY;
      for (int t = lane; t < nt; t += 32) mx = fmaxf(mx, pm[t]);
      mx = warp_max(mx);
      float sacc = 0.f;
      for (int t = lane; t < nt; t += 32) sacc += ps[t] * exp2f(pm[t] - mx);
      sacc = warp_sum(sacc);
      const float inv = 1.0f / (sacc * float(nbv));
      float* row = abar + size_t(qb) * nb;
      float* vrow = vals + qb * (qb + 1) / 2;
      for (int kb = lane; kb <= qb; kb += 32) {
        const float v = exp2f(row[kb] - mx) * inv;
        row[kb] = v;
        vrow[kb] = v;
      }
    }
  }
  if (tid == 0) st = PeState{};
  __syncthreads();
  // (2) radix select of the cut value, three levels
  const double g = double(p.gamma);
  for (int level = 0; level < 3; ++level) {
    int shift, nbk;
    level_geom(level, shift, nbk);
    for (int i = tid; i < nbk; i += kPeSmallThreads) { hc[i] = 0u; hs[i] = 0.0; }
    __syncthreads();
    const uint32_t hi_shift = shift + (level == 2 ? 8 : 12);
    const uint32_t prefix = st.prefix;
    for (int i0 = 0; i0 < M; i0 += kPeSmallThreads) {     // uniform trip count
      const int i = i0 + tid;
      bool take = false;
      uint32_t bk = 0xFFFFFFFFu;
      double sv = 0.0;
      if (i < M) {
        const float v = vals[i];
        const uint32_t u = __float_as_uint(v);
        if (level == 0 || (u >> hi_shift) == (prefix >> hi_shift)) {
          take = true;
          bk = (u >> shift) & uint32_t(nbk - 1);
          sv = double(v);
        }
      }
      hist_add_warp(hc, hs, take, bk, sv);
    }
    __syncthreads();
    // the highest bucket whose descending cumulative sum reaches gamma:
    // thread t owns the buckets counted from the top t*per .. t*per+per-1
    const int per = nbk / kPeSmallThreads > 0 ? nbk / kPeSmallThreads : 1;
    const int nact = nbk / per;
    double own = 0.0;
    if (tid < nact)
      for (int i = 0; i < per; ++i) own += hs[nbk - 1 - (tid * per + i)];
    scan[tid] = own;
    if (tid == 0) { ctl[0] = -1; ctl[1] = 1 << 30; }
    __syncthreads();
    for (int bkt = tid; bkt < nbk; bkt += kPeSmallThreads)
      if (hc[bkt]) atomicMin(&ctl[1], bkt);
    for (int off = 1; off < kPeSmallThreads; off <<= 1) {
      const double v = tid >= off ? scan[tid - off] : 0.0;
      __syncthreads();
      scan[tid] += v;
      __syncthreads();
    }
    const double above0 = st.above_sum;
    double run = above0 + (tid > 0 ? scan[tid - 1] : 0.0);
    int cand = -1;
    double cand_above = 0.0;
    if (tid < nact) {
      for (int i = 0; i < per; ++i) {
        const int bkt = nbk - 1 - (tid * per + i);
        const double v = hs[bkt];
        if (run + v >= g) { cand = bkt; cand_above = run; atomicMax(&ctl[0], bkt); break; }
        run += v;
      }
    }
    __syncthreads();
    if (cand >= 0 && cand == ctl[0]) scan[kPeSmallThreads] = cand_above;   // exactly one owner
    __syncthreads();
    if (tid == 0) {
      PeState s2 = st;
      const int best = ctl[0], lowest = ctl[1];
      int cut = best;
      if (cut < 0 && level > 0 && lowest < nbk) cut = lowest;   // rounding fell short: whole range
      if (cut < 0) {
        s2.all = 1;                                             // the whole triangle sums below gamma
      } else {
        const double above = cut == best ? scan[kPeSmallThreads] : above0 + scan[kPeSmallThreads - 1] - hs[cut];
        s2.prefix |= uint32_t(cut) << shift;
        s2.above_sum = above;
        if (level == 2) {
          const float tv = __uint_as_float(s2.prefix);
          const double need = g - above;
          double m = ceil(need / double(tv));
          if (m < 1.0) m = 1.0;
          const double cap = double(hc[cut]);
          if (m > cap) m = cap;
          s2.m_equal = uint32_t(m);
        }
      }
      st = s2;
    }
    __syncthreads();
    if (st.all) break;
  }
  // (3) per-row counts of entries equal to the cut value, exclusive scan
  if (!st.all) {
    const float tv = __uint_as_float(st.prefix);
    for (int qb = warp; qb < nbv; qb += kPeSmallThreads / 32) {
      const float* vrow = vals + qb * (qb + 1) / 2;
      uint32_t c = 0;
      for (int kb = lane; kb <= qb; kb += 32) c += vrow[kb] == tv;
      c = __reduce_add_sync(0xffffffffu, c);
      if (lane == 0) rowc[qb] = c;
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t* ec = ws_ptr<uint32_t>(ws, W.eq_cnt) + size_t(bh) * nb;
      uint32_t run = 0;
      for (int qb = 0; qb < nbv; ++qb) {
        const uint32_t c = rowc[qb];
        ec[qb] = run;
        run += c;
      }
    }
  }
  if (tid == 0) ws_ptr<PeState>(ws, W.pe_state)[bh] = st;
}

// ---------------------------------------------------------------------------
// Tile lists: one warp per (head, query block); a warp scan compacts the
// active ids in ascending order.
// VS: tile active iff kb in S_v u {0}, or a selected slash block (or N_b-1)
//     meets the tile: for a sequence whose length is a multiple of B, qb-kb
//     or qb-kb-1 in the offset set O = {N_b-1-j : j in S_s} u {0}; for a
//     partial last block see the rule below. Lanes take 32 key blocks each
//     from the selection bitmasks.
// PE: active iff chosen by the gamma cut, or kb == qb, or kb == 0; lanes take
//     4 consecutive key blocks per step.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) build_tiles_kernel(crisp_params p, const int32_t* pattern,
                                                          void* ws, uint8_t* __restrict__ mask,
                                                          int32_t* __restrict__ tile_idx,
                                                          int32_t* __restrict__ tile_cnt) {
  const Workspace W = make_workspace(p);
  const int nbs = n_blocks(p);                              // stride of the per-block arrays
  const int bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x * (blockDim.x >> 5) + warp;
  if (qb >= nbs) return;
  const int B = p.block;
  const int len = seq_len(p, bh / p.h_q);
  const int nb = (len + B - 1) / B;                         // this sequence's blocks
  int32_t* idx = tile_idx + (size_t(bh) * nbs + qb) * nbs;
  uint8_t* mrow = mask ? mask + (size_t(bh) * nbs + qb) * nbs : nullptr;
  if (qb >= nb) {                                           // past the end of a shorter sequence
    if (lane == 0) tile_cnt[size_t(bh) * nbs + qb] = 0;
    for (int j = lane; mrow && j < nbs; j += 32) mrow[j] = 0;
    return;
  }
  const bool vs = pattern[bh] == CRISP_PATTERN_VS;
  const uint8_t* sv = ws_ptr<uint8_t>(ws, W.sel) + size_t(bh) * 2 * nbs;
  const uint8_t* ss = sv + nbs;
  PeState st{};
  const float* arow = nullptr;
  uint32_t eq_before = 0;
  float tv = 0.f;
  if (!vs) {
    st = ws_ptr<PeState>(ws, W.pe_state)[bh];
    arow = ws_ptr<float>(ws, W.abar) + (size_t(bh) * nbs + qb) * nbs;
    tv = __uint_as_float(st.prefix);
    if (!st.all) eq_before = ws_ptr<uint32_t>(ws, W.eq_cnt)[size_t(bh) * nbs + qb];
  }
  // Slash blocks met by tile (qb, kb): pair (t, j) lies on slash index
  // j + len-1-t = (nb-1-delta) B + s + (c - r) with s = (len-1) mod B and
  // c - r over [-(rows(qb)-1), cols(kb)-1] (off the diagonal) or
  // [-(rows(qb)-1), 0] (on it); so the blocks nb-1-delta + {-1, 0, +1}
  // with the two ends decided by the signs below: -1 when some row of qb
  // lies past s (lo_ext), +1 off the diagonal when s >= 1. For len a
  // multiple of B this is {nb-1-delta, nb-delta}: offsets delta and delta-1.
  const int s_res = (len - 1) % B;
  const int rows_q = min(B, len - qb * B);
  const bool lo_ext = s_res - (rows_q - 1) < 0;
  auto slash_on = [&](int jb) -> bool { return jb == nb - 1 || (jb >= 0 && jb < nb && ss[jb] != 0); };
  // List entry of an active tile: the key-block id, plus in token
  // granularity the flags the attention kernel masks with (whole tile, or
  // which of the three slash blocks that can meet the tile are selected).
  const bool token = p.vs_granularity == CRISP_GRAN_TOKEN;
  auto tile_entry = [&](int kb) -> int32_t {
    if (!token) return kb;
    if (!vs || kb == 0 || sv[kb]) return kb | kTileWhole;
    int32_t v = kb;
    for (int e = -1; e <= 1; ++e)
      if (slash_on(nb - 1 - (qb - kb) + e)) v |= 1 << (kTileSlashShift + e + 1);
    return v;
  };

  if (vs) {
    // Vertical-slash row from the selection bitmasks, 32 key blocks per lane
    // word: kb is active iff it is a selected vertical block, or a selected
    // slash block jb = kb + c0 + t meets the tile, c0 = nb-1-qb and
    // t in [-1 if lo_ext, +1 if the bands reach the next block] (the slash
    // rule above, inverted).
    const int nw = (nbs + 31) / 32;
    const uint32_t* vwd = ws_ptr<uint32_t>(ws, W.sel_bits) + size_t(bh) * 2 * nw;
    const uint32_t* swd = vwd + nw;
    const int c0 = nb - 1 - qb;
    const bool up = s_res >= 1;                              // bands of full blocks reach jb + 1
    auto sword = [&](int wd, int sh) -> uint32_t {           // word wd of (S >> sh)
      const int base = wd * 32 + sh;
      const int q = base >> 5, rr = base & 31;
      const uint32_t lo = (q >= 0 && q < nw) ? swd[q] : 0u;
      const uint32_t hi = (q + 1 >= 0 && q + 1 < nw) ? swd[q + 1] : 0u;
      return rr ? (lo >> rr) | (hi << (32 - rr)) : lo;
    };
    const int nwq = (qb >> 5) + 1;                           // words holding kb <= qb
    int count = 0;
    for (int w0 = 0; w0 < nwq; w0 += 32) {
      const int wd = w0 + lane;
      uint32_t m = 0;
      if (wd < nwq) {
        m = vwd[wd] | sword(wd, c0);
        if (lo_ext) m |= sword(wd, c0 - 1);
        if (up) m |= sword(wd, c0 + 1);
        if (wd == nwq - 1 && (qb & 31) != 31) m &= (2u << (qb & 31)) - 1u;   // kb <= qb
      }
      const int c = __popc(m);
      int pre = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, pre, o);
        if (lane >= o) pre += v;
      }
      int pos = count + pre - c;
      for (uint32_t mm = m; mm; mm &= mm - 1) idx[pos++] = tile_entry(wd * 32 + __ffs(mm) - 1);
      if (mrow && wd < nwq)
        for (int i = 0; i < 32 && wd * 32 + i < nbs; ++i) mrow[wd * 32 + i] = (m >> i) & 1u;
      count += __shfl_sync(0xffffffffu, pre, 31);
    }
    for (int j = nwq * 32 + lane; mrow && j < nbs; j += 32) mrow[j] = 0;
    if (lane == 0) tile_cnt[size_t(bh) * nbs + qb] = count;
    return;
  }
  int count = 0;
  uint32_t eq_seen = eq_before;
  for (int base = 0; base <= qb; base += 128) {
    bool f[4];
    int neq = 0;
    bool isq[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int kb = base + lane * 4 + i;
      bool on = false;
      isq[i] = false;
      if (kb <= qb) {                                      // PE row (VS rows returned above)
        on = kb == 0 || kb == qb || st.all;
        if (!st.all) {
          const float v = arow[kb];
          if (v > tv) on = true;
          else if (v == tv) { isq[i] = true; ++neq; }
        }
      }
      f[i] = on;
    }
    if (!st.all) {
      // rank of this lane's equal entries among all equal entries in flat order
      uint32_t pre = neq;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, pre, o);
        if (lane >= o) pre += v;
      }
      uint32_t rank = eq_seen + pre - neq;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (isq[i]) { if (rank < st.m_equal) f[i] = true; ++rank; }
      eq_seen += __shfl_sync(0xffffffffu, pre, 31);
    }
    if (mrow) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (base + lane * 4 + i < nbs) mrow[base + lane * 4 + i] = f[i];
    }
    int c = int(f[0]) + int(f[1]) + int(f[2]) + int(f[3]);
    int pre = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, pre, o);
      if (lane >= o) pre += v;
    }
    int pos = count + pre - c;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (f[i]) idx[pos++] = tile_entry(base + lane * 4 + i);
    count += __shfl_sync(0xffffffffu, pre, 31);
    if (base + 128 > qb) {
      // the rest of the row lies above the diagonal: mask zeros only
      for (int b2 = base + 128 + lane; mrow && b2 < nbs; b2 += 32) mrow[b2] = 0;
      break;
    }
  }
  if (lane == 0) tile_cnt[size_t(bh) * nbs + qb] = count;
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
cudaError_t run_select(const crisp_params& p, const void* q, const void* k, const int32_t* pattern,
                       const float* p_v, const float* p_s, void* ws, uint8_t* mask,
                       int32_t* tile_idx, int32_t* tile_cnt, cudaStream_t st) {
  const Workspace W = make_workspace(p);
  const int nb = n_blocks(p);
  const int BH = p.batch * p.h_q;
  cudaError_t e;
  // (1) VS selection per direction.
  {
    const size_t smem = size_t(nb) * 8 + 1024 * 8;
    cudaFuncSetAttribute(vs_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    vs_select_kernel<<<dim3(BH, 2), 1024, smem, st>>>(p, pattern, p_v, p_s, ws);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // (2) PE path: pooling (K where the router has not pooled it already, Q of
  // PE heads), estimate, gamma cut (three radix levels, each with its cut
  // found by the last histogram CTA of the head), ties at the cut value.
  e = launch_pool(p, k, q, p.router == CRISP_ROUTER_JSD ? 0 : p.batch * p.h_kv, BH, pattern,
                  ws_ptr<float>(ws, W.kbar), ws_ptr<float>(ws, W.qbar), st);
  if (e != cudaSuccess) return e;
  {
    const int nt = (nb + 63) / 64;
    const unsigned grid = unsigned(min(nt * (nt + 1) / 2 * BH, 4 * 148));
    if (p.head_dim == 64) pe_logits_kernel<64><<<grid, 256, 0, st>>>(p, pattern, ws);
    else pe_logits_kernel<128><<<grid, 256, 0, st>>>(p, pattern, ws);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (size_t(nb) * (nb + 1) / 2 <= size_t(kPeSmallMax)) {
    // short sequences: normalisation, radix select and ties in one CTA per head
    e = cudaFuncSetAttribute(pe_small_cut_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kPeSmallSmem));
    if (e != cudaSuccess) return e;
    pe_small_cut_kernel<<<BH, kPeSmallThreads, kPeSmallSmem, st>>>(p, pattern, ws);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else {
    pe_normalize_kernel<<<dim3((nb + 7) / 8, BH), 256, 0, st>>>(p, pattern, ws);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    for (int level = 0; level < 3; ++level) {
      pe_hist_kernel<<<dim3((nb + 7) / 8, BH), 256, 0, st>>>(p, pattern, ws, level);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    pe_eqcount_kernel<<<dim3((nb + 7) / 8, BH), 256, 0, st>>>(p, pattern, ws);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // (3) tile lists.
  build_tiles_kernel<<<dim3((nb + 7) / 8, BH), 256, 0, st>>>(p, pattern, ws, mask, tile_idx, tile_cnt);
  return cudaGetLastError();
}

}  // namespace crisp
