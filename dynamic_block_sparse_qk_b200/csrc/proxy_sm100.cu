// Proxy attention statistics (CRISP paper, Algorithm 2, and the block scores
// that Algorithm 3 thresholds) on the 5th-generation tensor cores of sm_100a.
//
// The proxy rows are the last R = block query rows of a head. For every proxy
// row r and key tile kb this kernel writes the tile-local row max m (log2
// units) and the two partial sums of exp2(s - m) over the tile columns c <= r
// and c > r (the parts of the tile in slash blocks kb and kb + 1), plus, per
// chunk of proxy_chunk() key tiles, the running max / sum. The last CTA of a
// head to finish merges the chunks into each proxy row's max and normaliser.
// No b x n proxy map is ever stored.
//
// One CTA = one query head and one chunk of key tiles. The UMMA runs with
// M = 128 on the last 128 query rows (for block 64 the proxy rows are TMEM
// lanes 64..127) and N = 128 keys per step (one 128-key tile or two 64-key
// tiles):
//   warp 8 (one lane)  TMA producer: Q once, then the K tiles (ring).
//   warp 9 (one lane)  UMMA issuer: S_j = Q K_j^T into TMEM buffer j%2 once
//                      the softmax group has read S_{j-2}.
//   warps 0-3, 4-7     two row-statistics groups; group g takes the steps
//                      j with j%2 == g. Thread r owns TMEM lane r. The row max
//                      is one pass over the S row, the exp2 sums a second; in
//                      both the tile split c <= r / c > r is warp-uniform per
//                      32-column chunk except for the one chunk holding the
//                      diagonal.
// Two CTAs fit on an SM (256 TMEM columns and < 100 KB shared memory each).
// Every mbarrier wait is bounded (status CRISP_ERR_TIMEOUT and a CTA abort
// flag on expiry); the producer drains its copies and the issuer waits for a
// final commit of its UMMAs before the TMEM is released and the CTA exits.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace crisp {
using namespace sm100;

namespace {

constexpr int PM = 128;                  // UMMA M: query rows held in TMEM
constexpr int PN = 128;                  // keys per step (UMMA N)
constexpr int kPxThreads = 320;          // 2 x 4 statistics warps, producer, issuer
constexpr int kPxProd = 8, kPxMma = 9;
constexpr uint32_t kPxTmemCols = 256;    // S_0, S_1

template <int D>
struct PxCfg {
  static constexpr int NSLOT = D == 128 ? 2 : 4;
  static constexpr int Q_BYTES = PM * D * 2;
  static constexpr int T_BYTES = PN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = OFF_Q + Q_BYTES;
  static constexpr int OFF_XCH = OFF_RING + NSLOT * T_BYTES;    // float[2 groups][2][PM]
  static constexpr int OFF_BAR = OFF_XCH + 2 * 2 * PM * 4;
  static constexpr int B_Q = 0, B_KFULL = 1, B_KEMPTY = 1 + NSLOT, B_S = 1 + 2 * NSLOT, B_SFREE = B_S + 2,
                       B_DRAIN = B_SFREE + 2, N_BARS = B_DRAIN + 1;
  static constexpr int OFF_TMEM = OFF_BAR + 8 * N_BARS;
  static constexpr int OFF_ABORT = OFF_TMEM + 8;
  static constexpr int SMEM = OFF_ABORT + 8 + 1024;   // + alignment slack
  static_assert(2 * (SMEM + 1024) <= 233472, "two CTAs per SM");
};

// Proxy row max and normaliser of head bh from its nc chunk partials: one
// warp per row, lanes over chunks (fixed order: lane-strided partials, then a
// butterfly), so the loads of a row are in flight together. Out of line so
// that its addresses are not held in registers through the main loop.
__device__ __noinline__ void merge_chunks(const crisp_params& p, void* ws, int bh, int nc, int R) {
  const Workspace W = make_workspace(p);
  const float* cmv = ws_ptr<float>(ws, W.chunk_m) + size_t(bh) * nc * R;
  const float* clv = ws_ptr<float>(ws, W.chunk_l) + size_t(bh) * nc * R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int r = warp; r < R; r += nwarps) {
    float m = -INFINITY;
    for (int c = lane; c < nc; c += 32) m = fmaxf(m, __ldcg(cmv + size_t(c) * R + r));
    m = warp_max(m);
    float l = 0.f;
    for (int c = lane; c < nc; c += 32)
      l += __ldcg(clv + size_t(c) * R + r) * fast_exp2(__ldcg(cmv + size_t(c) * R + r) - m);
    l = warp_sum(l);
    if (lane == 0) {
      ws_ptr<float>(ws, W.row_m)[size_t(bh) * R + r] = m;
      ws_ptr<float>(ws, W.row_l)[size_t(bh) * R + r] = l;
    }
  }
}

template <int D, int R>
__global__ void __launch_bounds__(kPxThreads, 2)
    proxy_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    crisp_params p, void* ws, long long wait_limit) {
  using C = PxCfg<D>;
  constexpr int NSLOT = C::NSLOT;
  constexpr int KPS = PN / R;          // key tiles per step
  constexpr int ROW0 = PM - R;         // TMEM lane of proxy row 0
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_Q, sRing = base + C::OFF_RING;
  auto BAR = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * uint32_t(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_ABORT);

  const Workspace W = make_workspace(p);
  int32_t* status = ws_ptr<int32_t>(ws, W.status);
  const int N = p.seqlen, nb = n_blocks(p);
  const int chunk_tiles = proxy_chunk(p);
  const int nc = (nb + chunk_tiles - 1) / chunk_tiles;
  // CTA order: the query heads of one KV head are adjacent, so the CTAs that
  // run together stream the same K tiles (read from HBM once, then from L2).
  const int g = p.h_q / p.h_kv;
  const int hin = int(blockIdx.x) % g;
  const int t = int(blockIdx.x) / g;
  const int chunk = t % nc, bk = t / nc;          // bk = batch * h_kv + kv head
  const int b = bk / p.h_kv, hk = bk % p.h_kv;
  const int bh = b * p.h_q + hk * g + hin;
  // this sequence's length and blocks (chunks past its end have no steps)
  const int len = seq_len(p, b, (chunk == 0 && hin == 0 && hk == 0 && threadIdx.x == 0) ? status : nullptr);
  const int nbv = (len + R - 1) / R;
  const int kb0 = chunk * chunk_tiles, kb1 = min(kb0 + chunk_tiles, nbv);
  const int nsteps = kb1 > kb0 ? (kb1 - kb0 + KPS - 1) / KPS : 0;
  const int q_row = bh * N + len - PM;
  const int k_row0 = bk * N + kb0 * R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_Q), 1);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(BAR(C::B_KFULL + s), 1);
      mbar_init(BAR(C::B_KEMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::B_S + i), 1);
      mbar_init(BAR(C::B_SFREE + i), R / 32);   // one arrival per warp holding proxy rows
    }
    mbar_init(BAR(C::B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kPxMma) {
    tmem_alloc(smem_u32(tmem_slot), kPxTmemCols);
    tmem_relinquish();
  }
  if (warp == kPxProd && lane == 0) {
    prefetch_tmap(&tmq);
    prefetch_tmap(&tmk);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kPxProd) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(BAR(C::B_Q), C::Q_BYTES);
      for (int box = 0; box < D / 64; ++box) tma_load_2d(sQ + box * PM * 128, &tmq, box * 64, q_row, BAR(C::B_Q));
      int j = 0;
      for (; j < nsteps; ++j) {
        const int s = j % NSLOT, u = j / NSLOT;
        if (u >= 1 && !mbar_wait(BAR(C::B_KEMPTY + s), (u - 1) & 1, abort_flag, status, 21, wait_limit)) break;
        mbar_arrive_expect_tx(BAR(C::B_KFULL + s), C::T_BYTES);
        for (int box = 0; box < D / 64; ++box)
          tma_load_2d(sRing + s * C::T_BYTES + box * PN * 128, &tmk, box * 64, k_row0 + j * PN,
                      BAR(C::B_KFULL + s));
      }
      // no copy may still be landing when the CTA exits
      volatile int no_abort = 0;
      if (!mbar_test(BAR(C::B_Q), 0)) mbar_wait(BAR(C::B_Q), 0, &no_abort, status, 22, kDrainLimit);
      for (int s = 0; s < NSLOT && s < j; ++s) {
        const int last = s + ((j - 1 - s) / NSLOT) * NSLOT;
        if (!mbar_test(BAR(C::B_KFULL + s), (last / NSLOT) & 1))
          mbar_wait(BAR(C::B_KFULL + s), (last / NSLOT) & 1, &no_abort, status, 22, kDrainLimit);
      }
    }
  } else if (warp == kPxMma) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t idq = idesc_bf16(PM, PN, 0);
      bool ok = mbar_wait(BAR(C::B_Q), 0, abort_flag, status, 23, wait_limit);
      for (int j = 0; ok && j < nsteps; ++j) {
        if (j >= 2) {   // buffer j%2 is free once its group has read S_{j-2}
          ok = mbar_wait(BAR(C::B_SFREE + (j & 1)), ((j - 2) >> 1) & 1, abort_flag, status, 24, wait_limit);
          if (!ok) break;
        }
        const int s = j % NSLOT;
        ok = mbar_wait(BAR(C::B_KFULL + s), (j / NSLOT) & 1, abort_flag, status, 25, wait_limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(j & 1) * 128u;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * (PM * 128) + (kk & 3) * 32;
          const uint32_t boff = (kk >> 2) * (PN * 128) + (kk & 3) * 32;
          umma_ss(d, smem_desc_sw128(sQ + aoff, 16, 1024), smem_desc_sw128(sRing + s * C::T_BYTES + boff, 16, 1024),
                  idq, kk > 0);
        }
        umma_commit(BAR(C::B_S + (j & 1)));
        umma_commit(BAR(C::B_KEMPTY + s));
      }
      // Every UMMA issued here has completed before the TMEM is released
      // (after an abort some S_j may never have been read).
      umma_commit(BAR(C::B_DRAIN));
      volatile int no_abort = 0;
      mbar_wait(BAR(C::B_DRAIN), 0, &no_abort, status, 27, kDrainLimit);
    }
  } else if ((warp & 3) * 32 >= ROW0) {
    // ------------------------------------------------------------ row statistics
    const int grp = warp >> 2, quad = warp & 3;
    const int pr = quad * 32 + lane - ROW0;      // proxy row
    const int mixc = pr >> 5;                    // the 32-column chunk holding column pr (warp-uniform)
    const int prl = pr & 31;
    const uint32_t tS = tmem + (uint32_t(quad * 32) << 16) + uint32_t(grp) * 128u;
    const float sl2 = (p.sm_scale > 0.f ? p.sm_scale : rsqrtf(float(D))) * kLog2e;
    const uint64_t sc2 = pack_f32x2(sl2, sl2);
    float* stat_m = ws_ptr<float>(ws, W.stat_m);
    float* stat_lo = ws_ptr<float>(ws, W.stat_lo);
    float* stat_hi = ws_ptr<float>(ws, W.stat_hi);
    float cm = -INFINITY, cl = 0.f;

    // Columns past this row's causal limit `lim` (only in the last two key
    // tiles of a sequence) become -inf right after the TMEM load; the max and
    // sum passes below then need no masking of their own (exp2(-inf) = 0).
    auto mask_chunk = [&](uint32_t (&a)[32], int ci, int lim) {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (ci * 32 + e > lim) a[e] = 0xFF800000u;          // -inf
    };
    // exp2(s * sl2 - mx) summed over one 32-column chunk into lo (columns <= pr)
    // and hi (columns > pr); `ci` is the chunk index inside its key tile.
    auto chunk_sums = [&](const uint32_t (&a)[32], int ci, float mx, uint64_t& lo2, uint64_t& hi2) {
      const uint64_t nm2 = pack_f32x2(-mx, -mx);
      if (ci != mixc) {
        uint64_t acc2[2] = {pack_f32x2(0.f, 0.f), pack_f32x2(0.f, 0.f)};
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint64_t x2 = fma_f32x2(pack_f32x2(__uint_as_float(a[e]), __uint_as_float(a[e + 1])), sc2, nm2);
          float xa, xb;
          unpack_f32x2(x2, xa, xb);
          acc2[(e >> 1) & 1] = add_f32x2(acc2[(e >> 1) & 1], pack_f32x2(fast_exp2(xa), fast_exp2(xb)));
        }
        const uint64_t sum2 = add_f32x2(acc2[0], acc2[1]);
        if (ci < mixc) lo2 = add_f32x2(lo2, sum2);
        else hi2 = add_f32x2(hi2, sum2);
      } else {
        float lo = 0.f, hi = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float ex = fast_exp2(fmaf(__uint_as_float(a[e]), sl2, -mx));
          if (e <= prl) lo += ex;
          else hi += ex;
        }
        lo2 = add_f32x2(lo2, pack_f32x2(lo, 0.f));
        hi2 = add_f32x2(hi2, pack_f32x2(hi, 0.f));
      }
    };
    // max over one chunk (raw scores)
    auto chunk_max = [&](const uint32_t (&a)[32], float mx) -> float {
      float m2[2] = {mx, -INFINITY};
#pragma unroll
      for (int e = 0; e < 32; e += 2)
        m2[(e >> 1) & 1] = max3f(m2[(e >> 1) & 1], __uint_as_float(a[e]), __uint_as_float(a[e + 1]));
      return fmaxf(m2[0], m2[1]);
    };
    // A row with no visible key in the tile (possible in a partial last block)
    // stores max -inf and zero sums and leaves the running (max, sum) alone.
    auto finish_tile = [&](int kb, float mx, uint64_t lo2, uint64_t hi2) {
      float l0, l1, h0, h1;
      unpack_f32x2(lo2, l0, l1);
      unpack_f32x2(hi2, h0, h1);
      const bool any = mx != -INFINITY;
      const float lo = any ? l0 + l1 : 0.f, hi = any ? h0 + h1 : 0.f;
      const size_t o = (size_t(bh) * nb + kb) * R + pr;
      stat_m[o] = mx;
      stat_lo[o] = lo;
      stat_hi[o] = hi;
      if (any) {
        const float nm = fmaxf(cm, mx);
        cl = cl * fast_exp2(cm - nm) + (lo + hi) * fast_exp2(mx - nm);
        cm = nm;
      }
    };
    const int t_row = len - R + pr;            // position of this proxy row

    int u = 0;
    for (int j = grp; j < nsteps; j += 2, ++u) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(BAR(C::B_S + grp), u & 1, abort_flag, status, 26, wait_limit));
      if (!ok) break;
      tc_fence_after();
      const int kbs = kb0 + j * KPS;
      uint32_t a0[32], a1[32];
      if constexpr (R == 64) {
        // two 64-key tiles per step, each one pair of chunks loaded once
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          tmem_ld32(tS + ks * 64, a0);
          tmem_ld32(tS + ks * 64 + 32, a1);
          tmem_wait_ld();
          if (ks == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(C::B_SFREE + grp));
          }
          const int kb = kbs + ks;
          if (kb < kb1) {
            if (kb >= nbv - 2) {                         // causal limit inside the tile
              const int lim = t_row - kb * R;
              mask_chunk(a0, 0, lim);
              mask_chunk(a1, 1, lim);
            }
            float mx = chunk_max(a0, -INFINITY);
            mx = chunk_max(a1, mx) * sl2;
            uint64_t lo2 = pack_f32x2(0.f, 0.f), hi2 = pack_f32x2(0.f, 0.f);
            if (mx != -INFINITY) {
              chunk_sums(a0, 0, mx, lo2, hi2);
              chunk_sums(a1, 1, mx, lo2, hi2);
            }
            finish_tile(kb, mx, lo2, hi2);
          }
        }
      } else {
        // one 128-key tile: a max pass and a sum pass over two pairs of chunks
        const int kb = kbs;
        const bool masked = kb >= nbv - 2;               // causal limit inside the tile
        const int lim = t_row - kb * R;
        tmem_ld32(tS, a0);
        tmem_ld32(tS + 32, a1);
        tmem_wait_ld();
        if (masked) {
          mask_chunk(a0, 0, lim);
          mask_chunk(a1, 1, lim);
        }
        float mx = chunk_max(a0, -INFINITY);
        mx = chunk_max(a1, mx);
        uint32_t a2[32], a3[32];
        tmem_ld32(tS + 64, a2);
        tmem_ld32(tS + 96, a3);
        tmem_wait_ld();
        if (masked) {
          mask_chunk(a2, 2, lim);
          mask_chunk(a3, 3, lim);
        }
        mx = chunk_max(a2, mx);
        mx = chunk_max(a3, mx) * sl2;
        uint64_t lo2 = pack_f32x2(0.f, 0.f), hi2 = pack_f32x2(0.f, 0.f);
        const bool any = mx != -INFINITY;
        if (any) {
          chunk_sums(a2, 2, mx, lo2, hi2);
          chunk_sums(a3, 3, mx, lo2, hi2);
        }
        tmem_ld32(tS, a0);
        tmem_ld32(tS + 32, a1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_SFREE + grp));
        if (masked) {
          mask_chunk(a0, 0, lim);
          mask_chunk(a1, 1, lim);
        }
        if (any) {
          chunk_sums(a0, 0, mx, lo2, hi2);
          chunk_sums(a1, 1, mx, lo2, hi2);
        }
        finish_tile(kb, mx, lo2, hi2);
      }
    }
    // ---- merge the two groups' running (max, sum) for this chunk (every
    // statistics thread gets here exactly once)
    float* xch = reinterpret_cast<float*>(gbase + C::OFF_XCH);
    xch[(grp * 2) * PM + pr] = cm;
    xch[(grp * 2 + 1) * PM + pr] = cl;
    asm volatile("bar.sync 1, %0;" ::"r"(2 * R) : "memory");
    if (grp == 0) {
      const float m1 = xch[2 * PM + pr], l1 = xch[3 * PM + pr];
      float m = cm, l = cl;
      if (m1 != -INFINITY) {
        if (m == -INFINITY) {
          m = m1;
          l = l1;
        } else {
          const float mm = fmaxf(m, m1);
          l = l * fast_exp2(m - mm) + l1 * fast_exp2(m1 - mm);
          m = mm;
        }
      }
      const size_t o = (size_t(bh) * nc + chunk) * R + pr;
      ws_ptr<float>(ws, W.chunk_m)[o] = m;
      ws_ptr<float>(ws, W.chunk_l)[o] = l;
    }
  }

  __threadfence();      // this CTA's statistics are visible device-wide before it is counted
  tc_fence_before();
  __syncthreads();
  if (warp == kPxMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kPxTmemCols);
  }

  // ---- the last CTA of this head merges the chunk partials into the proxy
  // row max and normaliser (fixed chunk order: the result does not depend on
  // which CTA finishes last)
  volatile int* last = reinterpret_cast<volatile int*>(gbase + C::OFF_ABORT) + 1;
  uint32_t* cnt = ws_ptr<uint32_t>(ws, make_workspace(p).head_cnt) + size_t(bh) * 4 + kCntProxy;
  if (threadIdx.x == 0) *last = atomicAdd(cnt, 1u) == uint32_t(nc - 1);
  __syncthreads();
  if (!*last) return;
  __threadfence();
  merge_chunks(p, ws, bh, nc, R);
  if (threadIdx.x == 0) *cnt = 0u;   // ready for the next call
}

template <int D, int R>
cudaError_t launch_proxy(const crisp_params& p, const void* q, const void* k, void* ws, cudaStream_t st,
                         long long wait_limit) {
  CUtensorMap mq, mk;
  const uint64_t N = uint64_t(p.seqlen);
  if (!make_tmap(&mq, q, uint64_t(p.batch) * p.h_q * N, D) || !make_tmap(&mk, k, uint64_t(p.batch) * p.h_kv * N, D))
    return cudaErrorInvalidValue;
  auto kern = proxy_tc_kernel<D, R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PxCfg<D>::SMEM);
  if (e != cudaSuccess) return e;
  const int nb = n_blocks(p);
  const int nc = (nb + proxy_chunk(p) - 1) / proxy_chunk(p);
  const unsigned grid = unsigned(p.batch) * p.h_q * nc;
  kern<<<grid, kPxThreads, PxCfg<D>::SMEM, st>>>(mq, mk, p, ws, wait_limit);
  return cudaGetLastError();
}

}  // namespace

cudaError_t run_proxy_stats(const crisp_params& p, const void* q, const void* k, void* ws, cudaStream_t st,
                            long long wait_limit) {
  const long long wl = wait_limit;
  if (p.head_dim == 64)
    return p.block == 64 ? launch_proxy<64, 64>(p, q, k, ws, st, wl) : launch_proxy<64, 128>(p, q, k, ws, st, wl);
  return p.block == 64 ? launch_proxy<128, 64>(p, q, k, ws, st, wl) : launch_proxy<128, 128>(p, q, k, ws, st, wl);
}

}  // namespace crisp
