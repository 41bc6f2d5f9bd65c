// Block-sparse causal GQA flash attention (CRISP paper, Eq. 1) on the
// 5th-generation tensor cores of sm_100a.
//
// One CTA = one 128-row query tile of one head; it walks the 128-key tiles
// that the tile lists select (the union over the query blocks the tile covers,
// with a per-block membership mask), in ascending order: steps j = 0..n-1.
//
//   warp 8 (one lane)  TMA producer of Q and of the K tiles (a ring of 2
//                      slots for d = 128, 4 for d = 64).
//   warp 10 (one lane) TMA producer of the V tiles (a ring of the same depth).
//   warp 9 (one lane)  UMMA issuer of S_j = Q K_j^T into TMEM buffer j%2, as
//                      soon as the softmax has read S_{j-2} from that buffer.
//   warp 11 (one lane) UMMA issuer of O_{j%2} += P_j V_j into one of two TMEM
//                      accumulators, as soon as P_j is written. The two issuers
//                      touch disjoint buffers, so a late V tile never holds up
//                      the next QK^T and vice versa.
//   Work order: KV-head major, longest query tiles first within a KV head.
//   warps 0-3, 4-7     two softmax groups that ping-pong: group g takes the
//                      steps j with j%2 == g, so one group's exp2 work overlaps
//                      the other group's TMEM loads, stores and barriers.
//                      Thread r of a group owns query row r (TMEM lane r):
//                      tcgen05.ld of S, causal / block mask as one column
//                      window, row max, exp2, P written as bf16 into its
//                      group's swizzled shared tile for the PV UMMA; each group
//                      keeps its own running max m_g and sum l_g and rescales
//                      its accumulator in TMEM only when m_g grows by more
//                      than 2^8. At the end the two partial results merge:
//                      O = (O_0 2^(m_0-M) + O_1 2^(m_1-M)) / (l_0 2^(m_0-M) + l_1 2^(m_1-M)).
//
// Every mbarrier wait is bounded; a wait that runs out records
// CRISP_ERR_TIMEOUT in the workspace status word and raises a CTA abort flag,
// after which all roles leave their loops, the producers wait (bounded) for
// their copies in flight, each UMMA issuer waits (bounded) for a final commit
// of everything it issued, and only then is the TMEM allocation released.
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace crisp {
using namespace sm100;

namespace {

constexpr int BM = 128;          // query rows per CTA (UMMA M)
constexpr int BN = 128;          // keys per step (UMMA N of QK^T)
constexpr int kThreads = 384;    // 2 x 4 softmax warps, 2 producer warps, 2 UMMA warps
constexpr int kKProdWarp = 8, kSWarp = 9, kVProdWarp = 10, kPVWarp = 11;
constexpr uint32_t kTmemCols = 512;  // S_0, S_1 (128 each), O_0, O_1 (D each)

template <int D>
struct Cfg {
  static constexpr int NSLOT = D == 128 ? 2 : 4;          // per ring (K and V)
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int P_BYTES = BM * BN * 2;          // one group's P tile
  static constexpr int T_BYTES = BN * D * 2;           // one K or V tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = OFF_Q + Q_BYTES;
  static constexpr int OFF_RING = OFF_P + 2 * P_BYTES;
  static constexpr int OFF_VRING = OFF_RING + NSLOT * T_BYTES;
  static constexpr int OFF_BAR = OFF_VRING + NSLOT * T_BYTES;
  static constexpr int B_Q = 0, B_KFULL = 1, B_KEMPTY = 1 + NSLOT, B_VFULL = 1 + 2 * NSLOT,
                       B_VEMPTY = 1 + 3 * NSLOT, B_S = 1 + 4 * NSLOT, B_SFREE = B_S + 2,
                       B_P = B_SFREE + 2, B_PV = B_P + 2, B_O = B_PV + 2, B_SDRAIN = B_O + 1,
                       N_BARS = B_SDRAIN + 1;
  static constexpr int OFF_TMEM = OFF_BAR + 8 * N_BARS;
  static constexpr int OFF_ABORT = OFF_TMEM + 8;
  static constexpr int SMEM = OFF_ABORT + 8 + 1024;   // + alignment slack
  static_assert(SMEM <= 232448, "shared memory budget");
};

// Walks the 128-key tiles a query tile needs, ascending, with membership bits:
// bit (i * kpu + ks) says query block qb0+i attends key block kt*kpu+ks.
// Bits 8..11 carry the token-granularity flags of the tile (bit 8: whole
// tile; bits 9..11: slash blocks N_b-1-delta+e selected, e = -1, 0, +1); a
// dense walk, tile-granularity lists and 64-wide blocks mark every tile whole.
constexpr uint32_t kStepWhole = 1u << 8;
struct StepIter {
  const int32_t* lst[2];
  int cnt[2], pos[2];
  int nsub, kpu, qb0, dense_last, next_kt;
  int ahead;        // single list: the next entry, already loaded (-2: none)
  int32_t* status;
  bool report, token;

  __device__ void init(const int32_t* tile_idx, const int32_t* tile_cnt, int bh, int nb, int block,
                       int qt, int32_t* st, bool rep, bool tok) {
    nsub = BM / block;
    kpu = BN / block;
    qb0 = qt * nsub;
    status = st;
    report = rep;
    token = tok && nsub == 1;
    next_kt = 0;
    dense_last = tile_idx ? -1 : qt;
    for (int i = 0; i < 2; ++i) { lst[i] = nullptr; cnt[i] = 0; pos[i] = 0; }
    if (tile_idx) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        if (i >= nsub) break;
        const int qb = qb0 + i;
        if (qb >= nb) break;                 // a 64-wide block past the stored rows
        lst[i] = tile_idx + (size_t(bh) * nb + qb) * nb;
        int c = tile_cnt[size_t(bh) * nb + qb];
        if (c < 0 || c > qb + 1) {
          if (report) report_error(status, CRISP_ERR_DEVICE, c);
          c = c < 0 ? 0 : qb + 1;
        }
        cnt[i] = c;
      }
    }
    ahead = -2;
    if (tile_idx && nsub == 1 && cnt[0] > 0) ahead = lst[0][0];
  }

  __device__ bool next(int& kt, uint32_t& bits) {
    if (dense_last >= 0) {
      if (next_kt > dense_last) return false;
      kt = next_kt++;
      bits = kStepWhole;
      for (int i = 0; i < nsub; ++i)
        for (int ks = 0; ks < kpu; ++ks)
          if (kt * kpu + ks <= qb0 + i) bits |= 1u << (i * kpu + ks);
      return true;
    }
    if (nsub == 1) {
      // one list: the entry was loaded on the previous call, load the next now
      while (pos[0] < cnt[0]) {
        const int v = ahead;
        ++pos[0];
        ahead = pos[0] < cnt[0] ? lst[0][pos[0]] : -2;
        const int id = token ? (v & kTileIdMask) : v;
        if (v >= 0 && id <= qb0) {
          kt = id / kpu;
          bits = (1u << (id % kpu)) | (token ? ((uint32_t(v) >> 24) & 15u) << 8 : kStepWhole);
          return true;
        }
        if (report) report_error(status, CRISP_ERR_DEVICE, v);
      }
      return false;
    }
    int best = INT_MAX;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (i >= nsub) break;
      while (pos[i] < cnt[i]) {
        const int v = lst[i][pos[i]];
        if (v >= 0 && v <= qb0 + i) break;
        if (report) report_error(status, CRISP_ERR_DEVICE, v);
        ++pos[i];
      }
      if (pos[i] < cnt[i]) best = min(best, lst[i][pos[i]] / kpu);
    }
    if (best == INT_MAX) return false;
    bits = kStepWhole;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (i >= nsub) break;
      while (pos[i] < cnt[i]) {
        const int v = lst[i][pos[i]];
        if (v < 0 || v > qb0 + i) {
          if (report) report_error(status, CRISP_ERR_DEVICE, v);
          ++pos[i];
          continue;
        }
        if (v / kpu != best) break;
        bits |= 1u << (i * kpu + v % kpu);
        ++pos[i];
      }
    }
    kt = best;
    return true;
  }
};

template <int D, int BLK, bool TOKEN>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv, const int32_t* __restrict__ tile_idx,
                   const int32_t* __restrict__ tile_cnt, __nv_bfloat16* __restrict__ o,
                   float* __restrict__ lse, crisp_params p, void* ws, long long wait_limit) {
  using C = Cfg<D>;
  constexpr int NSLOT = C::NSLOT;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_Q, sP = base + C::OFF_P, sRing = base + C::OFF_RING;
  const uint32_t sVRing = base + C::OFF_VRING;
  auto BAR = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * uint32_t(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_ABORT);

  const Workspace W = make_workspace(p);
  int32_t* status = ws_ptr<int32_t>(ws, W.status);
  const int N = p.seqlen, nb = n_blocks(p), NT = (N + BM - 1) / BM;
  constexpr bool token = TOKEN;   // token-granular slash bands (block 128 lists only)
  // Work order: KV-head major (the CTAs running at the same time read the same
  // K/V stream, which then stays in L2), longest query tiles first inside.
  const int g = p.h_q / p.h_kv;
  const int grp_items = g * NT;
  const int bk = int(blockIdx.x) / grp_items;         // batch * h_kv + kv head
  const int rem = int(blockIdx.x) % grp_items;
  const int qt = NT - 1 - rem / g;
  const int b = bk / p.h_kv, hk = bk % p.h_kv, h = hk * g + rem % g;
  const int bh = b * p.h_q + h;
  const int row0 = qt * BM;
  const int q_row = bh * N + row0;
  const int kv_row0 = (b * p.h_kv + hk) * N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // This sequence's length: a query tile wholly past it only writes its
  // stored rows as zeros (lse -inf).
  const int len = seq_len(p, b, (qt == 0 && h == 0 && threadIdx.x == 0) ? status : nullptr);
  if (row0 >= len) {
    const int rows = min(BM, N - row0);
    for (int i = threadIdx.x; i < rows * (D / 8); i += kThreads)
      reinterpret_cast<uint4*>(o + (size_t(bh) * N + row0) * D)[i] = make_uint4(0, 0, 0, 0);
    if (lse)
      for (int i = threadIdx.x; i < rows; i += kThreads) lse[size_t(bh) * N + row0 + i] = -INFINITY;
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_Q), 1);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(BAR(C::B_KFULL + s), 1);
      mbar_init(BAR(C::B_KEMPTY + s), 1);
      mbar_init(BAR(C::B_VFULL + s), 1);
      mbar_init(BAR(C::B_VEMPTY + s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(BAR(C::B_S + g), 1);
      mbar_init(BAR(C::B_SFREE + g), 4);   // one arrival per warp of group g
      mbar_init(BAR(C::B_P + g), 4);
      mbar_init(BAR(C::B_PV + g), 1);
    }
    mbar_init(BAR(C::B_O), 1);
    mbar_init(BAR(C::B_SDRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kSWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp == kKProdWarp && lane == 0) {
    prefetch_tmap(&tmq);
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kKProdWarp || warp == kVProdWarp) {
    // ------------------------------------------------------------ TMA producers
    if (lane == 0) {
      const bool is_k = warp == kKProdWarp;
      const CUtensorMap* map = is_k ? &tmk : &tmv;
      const uint32_t ring = is_k ? sRing : sVRing;
      const int bfull = is_k ? C::B_KFULL : C::B_VFULL, bempty = is_k ? C::B_KEMPTY : C::B_VEMPTY;
      StepIter it;
      it.init(tile_idx, tile_cnt, bh, nb, BLK, qt, status, is_k, token);
      if (is_k) {
        mbar_arrive_expect_tx(BAR(C::B_Q), C::Q_BYTES);
        for (int box = 0; box < D / 64; ++box)
          tma_load_2d(sQ + box * BM * 128, &tmq, box * 64, q_row, BAR(C::B_Q));
      }
      int t = 0, kt;
      uint32_t bits;
      while (it.next(kt, bits)) {
        const int s = t % NSLOT, u = t / NSLOT;
        if (u >= 1 && !mbar_wait(BAR(bempty + s), (u - 1) & 1, abort_flag, status, 1, wait_limit)) break;
        mbar_arrive_expect_tx(BAR(bfull + s), C::T_BYTES);
        for (int box = 0; box < D / 64; ++box)
          tma_load_2d(ring + s * C::T_BYTES + box * BN * 128, map, box * 64, kv_row0 + kt * BN, BAR(bfull + s));
        ++t;
      }
      // no copy may still be landing when the CTA exits (Q included)
      volatile int no_abort = 0;
      if (is_k && !mbar_test(BAR(C::B_Q), 0)) mbar_wait(BAR(C::B_Q), 0, &no_abort, status, 2, kDrainLimit);
      for (int s = 0; s < NSLOT && s < t; ++s) {
        const int last = s + ((t - 1 - s) / NSLOT) * NSLOT;
        if (!mbar_test(BAR(bfull + s), (last / NSLOT) & 1))
          mbar_wait(BAR(bfull + s), (last / NSLOT) & 1, &no_abort, status, 2, kDrainLimit);
      }
    }
  } else if (warp == kSWarp) {
    // ------------------------------------------------------------ UMMA issuer: S_j = Q K_j^T
    if (lane == 0) {
      StepIter it;
      it.init(tile_idx, tile_cnt, bh, nb, BLK, qt, status, false, token);
      constexpr uint32_t idq = idesc_bf16(BM, BN, 0);
      bool ok = mbar_wait(BAR(C::B_Q), 0, abort_flag, status, 4, wait_limit);
      int j = 0, kt;
      uint32_t bits;
      while (ok && it.next(kt, bits)) {
        if (j >= 2) {   // buffer j%2 is free once its softmax group has read S_{j-2}
          ok = mbar_wait(BAR(C::B_SFREE + (j & 1)), ((j - 2) >> 1) & 1, abort_flag, status, 5, wait_limit);
          if (!ok) break;
        }
        const int s = j % NSLOT;
        ok = mbar_wait(BAR(C::B_KFULL + s), (j / NSLOT) & 1, abort_flag, status, 3, wait_limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(j & 1) * 128u;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          const uint32_t boff = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
          umma_ss(d, smem_desc_sw128(sQ + aoff, 16, 1024),
                  smem_desc_sw128(sRing + s * C::T_BYTES + boff, 16, 1024), idq, kk > 0);
        }
        umma_commit(BAR(C::B_S + (j & 1)));
        umma_commit(BAR(C::B_KEMPTY + s));
        ++j;
      }
      // Every QK^T this lane issued has completed before the TMEM is released
      // (after an abort some S_j may never have been read).
      umma_commit(BAR(C::B_SDRAIN));
      volatile int no_abort = 0;
      mbar_wait(BAR(C::B_SDRAIN), 0, &no_abort, status, 11, kDrainLimit);
    }
  } else if (warp == kPVWarp) {
    // ------------------------------------------------------------ UMMA issuer: O += P V
    if (lane == 0) {
      StepIter it;
      it.init(tile_idx, tile_cnt, bh, nb, BLK, qt, status, false, token);
      constexpr uint32_t idp = idesc_bf16(BM, D, 1);
      bool ok = true;
      int j = 0, kt;
      uint32_t bits;
      while (ok && it.next(kt, bits)) {
        const int s = j % NSLOT;
        ok = mbar_wait(BAR(C::B_VFULL + s), (j / NSLOT) & 1, abort_flag, status, 3, wait_limit) &&
             mbar_wait(BAR(C::B_P + (j & 1)), (j >> 1) & 1, abort_flag, status, 6, wait_limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + 256u + uint32_t(j & 1) * D;
        const uint32_t pb = sP + uint32_t(j & 1) * C::P_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          const uint32_t boff = kk * (16 * 128);
          umma_ss(d, smem_desc_sw128(pb + aoff, 16, 1024),
                  smem_desc_sw128(sVRing + s * C::T_BYTES + boff, BN * 128, 1024), idp,
                  (j >= 2 || kk > 0) ? 1u : 0u);
        }
        umma_commit(BAR(C::B_PV + (j & 1)));
        umma_commit(BAR(C::B_VEMPTY + s));
        ++j;
      }
      umma_commit(BAR(C::B_O));
      // every PV this lane issued has completed before the TMEM is released
      volatile int no_abort = 0;
      mbar_wait(BAR(C::B_O), 0, &no_abort, status, 12, kDrainLimit);
    }
  } else {
    // ------------------------------------------------------------ softmax groups
    const int grp = warp >> 2, quad = warp & 3;
    const int r = quad * 32 + lane;               // query row within the tile = TMEM lane
    const int row = row0 + r;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + uint32_t(grp) * 128u;
    const uint32_t tO0 = tmem + lane_off + 256u;  // O_0; O_1 at + D
    const uint32_t tO = tO0 + uint32_t(grp) * D;
    const uint32_t prow = sP + uint32_t(grp) * C::P_BYTES + uint32_t(r) * 128u;
    constexpr int kpu = BN / BLK;
    constexpr uint32_t kmask = (1u << kpu) - 1u;
    const int qsub = r / BLK;
    const float sl2 = (p.sm_scale > 0.f ? p.sm_scale : rsqrtf(float(D))) * kLog2e;
    StepIter it;
    it.init(tile_idx, tile_cnt, bh, nb, BLK, qt, status, false, token);
    float m_use = -INFINITY, l = 0.f;
    int j = grp, u = 0, kt, kt_next;
    uint32_t bits, bits_next;
    bool ok = true;
    // this group's steps are j = grp, grp + 2, ...: the tile id and mask bits of
    // the next one are fetched while the current one is processed
    bool more = it.next(kt_next, bits_next) && (grp == 0 || it.next(kt_next, bits_next));
    while (more) {
      kt = kt_next;
      bits = bits_next;
      more = it.next(kt_next, bits_next) && it.next(kt_next, bits_next);
      ok = __all_sync(0xffffffffu, mbar_wait(BAR(C::B_S + grp), u & 1, abort_flag, status, 7, wait_limit));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_SFREE + grp));      // S buffer may be overwritten
      // Allowed key columns form one window [lo, hi]: the causal limit row - key0
      // and, for 64-wide blocks, which halves of the key tile this row's query
      // block selected.
      const uint32_t rb = (bits >> (qsub * kpu)) & kmask;
      const int lim = row - kt * BN;
      int lo = 0, hi = lim < BN - 1 ? lim : BN - 1;
      if (kpu == 2) {
        if (!(rb & 1u)) lo = BLK;
        if (!(rb & 2u)) hi = min(hi, BLK - 1);
      } else if (!rb) {
        hi = -1;
      }
      if (TOKEN && !(bits & kStepWhole)) {
        // Token granularity (block 128): only the diagonal bands of the
        // selected slash blocks N_b-1-delta+e, e = -1, 0, +1; for this row the
        // band of e covers columns [r - s + e B, r - s + e B + B - 1],
        // s = (len - 1) mod B. Inside the tile the bands e = -1 and e = +1
        // exclude each other (the first needs r > s, the second r < s), so
        // the selected bands always leave one window per row.
        const uint32_t f = (bits >> 9) & 7u;
        const int s_res = (len - 1) & (BLK - 1);
        const int a = r - s_res - BN;
        int wlo = 1, whi = 0;
        if (f == 5u) {
          wlo = r > s_res ? a : a + 2 * BN;
          whi = wlo + BN - 1;
        } else if (f) {
          wlo = a + (__ffs(f) - 1) * BN;
          whi = a + (32 - __clz(f)) * BN - 1;
        }
        lo = max(lo, wlo);
        hi = min(hi, whi);
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (lo == 0 && hi == BN - 1) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            mx[(e >> 1) & 3] = max3f(mx[(e >> 1) & 3], __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int col = c * 32 + e;
            const float x = (col >= lo && col <= hi) ? __uint_as_float(sr[c][e]) : -INFINITY;
            sr[c][e] = __float_as_uint(x);
            mx[e & 3] = fmaxf(mx[e & 3], x);
          }
      }
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
      float factor = 1.f;
      bool resc = false;
      if (u == 0) {
        m_use = mt;                      // the first step of either group has a visible key
      } else if (mt > m_use + 8.f) {
        factor = fast_exp2(m_use - mt);
        m_use = mt;
        resc = true;
      }
      const float mref = m_use == -INFINITY ? 0.f : m_use;
      // this group's P tile and O accumulator are free once its PV of step j-2 completed
      if (u >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(BAR(C::B_PV + grp), (u - 1) & 1, abort_flag, status, 8, wait_limit));
        if (!ok) break;
      }
      // exp2 arguments and row sums two at a time (f32x2), P packed to bf16x2
      const uint64_t sc2 = pack_f32x2(sl2, sl2), nm2 = pack_f32x2(-mref, -mref);
      uint64_t acc2[2] = {pack_f32x2(0.f, 0.f), pack_f32x2(0.f, 0.f)};
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {          // 16-byte chunk = 8 keys
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint64_t x2 = fma_f32x2(pack_f32x2(__uint_as_float(sr[ch >> 2][(ch & 3) * 8 + 2 * e]),
                                                   __uint_as_float(sr[ch >> 2][(ch & 3) * 8 + 2 * e + 1])),
                                        sc2, nm2);
          float xa, xb;
          unpack_f32x2(x2, xa, xb);
          const float a = fast_exp2(xa), bq = fast_exp2(xb);
          acc2[e & 1] = add_f32x2(acc2[e & 1], pack_f32x2(a, bq));
          pk[e] = pack_bf16(a, bq);
        }
        const uint32_t addr = prow + uint32_t(ch >> 3) * (BM * 128) + (uint32_t((ch & 7) ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(pk[0]), "r"(pk[1]),
                     "r"(pk[2]), "r"(pk[3])
                     : "memory");
      }
      float r0, r1, r2, r3;
      unpack_f32x2(acc2[0], r0, r1);
      unpack_f32x2(acc2[1], r2, r3);
      l = l * factor + ((r0 + r1) + (r2 + r3));
      if (__any_sync(0xffffffffu, resc)) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(tO + c * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * factor);
          tmem_st32(tO + c * 32, ov);
        }
        tmem_wait_st();
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_P + grp));
      j += 2;
      ++u;
    }
    // ---- merge the two groups' partial results (every softmax thread gets here once)
    const bool done = ok && __all_sync(0xffffffffu, mbar_wait(BAR(C::B_O), 0, abort_flag, status, 10, wait_limit));
    // all UMMAs have completed: the P tiles are free and hold the exchange
    float* xch = reinterpret_cast<float*>(gbase + C::OFF_P);
    xch[grp * 256 + r] = done ? m_use : -INFINITY;
    xch[grp * 256 + 128 + r] = done ? l : 0.f;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    const float m0 = xch[r], l0 = xch[128 + r], m1 = xch[256 + r], l1 = xch[384 + r];
    const float mm = fmaxf(m0, m1);
    const float w0 = l0 > 0.f ? fast_exp2(m0 - mm) : 0.f;
    const float w1 = l1 > 0.f ? fast_exp2(m1 - mm) : 0.f;
    const float lt = l0 * w0 + l1 * w1;
    __nv_bfloat16* orow = o + (size_t(bh) * N + row) * D + grp * (D / 2);
    // rows past the sequence (padding, or the next head's rows when the tile
    // runs past seqlen) never decide the warp's path; stored padding rows are zero
    const bool mine = row < len, stored = row < N;
    const bool fin = __all_sync(0xffffffffu, done && (!mine || lt > 0.f));
    if (fin) {
      tc_fence_after();
      const float a0 = w0 / lt, a1 = w1 / lt;
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        const uint32_t col = uint32_t(grp) * (D / 2) + c * 32;
        uint32_t v0[32], v1[32];
        tmem_ld32(tO0 + col, v0);
        tmem_ld32(tO0 + D + col, v1);
        tmem_wait_ld();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x0 = a0 != 0.f ? __uint_as_float(v0[q4 * 8 + e]) * a0 : 0.f;
            const float x1 = a1 != 0.f ? __uint_as_float(v1[q4 * 8 + e]) * a1 : 0.f;
            f[e] = x0 + x1;
          }
          uint4 pk = make_uint4(0, 0, 0, 0);
          if (mine) {
            pk.x = pack_bf16(f[0], f[1]);
            pk.y = pack_bf16(f[2], f[3]);
            pk.z = pack_bf16(f[4], f[5]);
            pk.w = pack_bf16(f[6], f[7]);
          }
          if (stored) *reinterpret_cast<uint4*>(orow + c * 32 + q4 * 8) = pk;
        }
      }
      if (lse && grp == 0 && stored) lse[size_t(bh) * N + row] = mine ? (mm + log2f(lt)) * kLn2 : -INFINITY;
    } else if (stored) {
      for (int c = 0; c < D / 2; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
      if (lse && grp == 0) lse[size_t(bh) * N + row] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kSWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ----------------------------------------------------------------------------- host
template <int D, int BLK, bool TOKEN>
cudaError_t launch_tc(const crisp_params& p, const void* q, const void* k, const void* v,
                      const int32_t* tile_idx, const int32_t* tile_cnt, void* o, float* lse, void* ws,
                      cudaStream_t st, long long wait_limit) {
  CUtensorMap mq, mk, mv;
  const uint64_t N = uint64_t(p.seqlen);
  if (!make_tmap(&mq, q, uint64_t(p.batch) * p.h_q * N, D) || !make_tmap(&mk, k, uint64_t(p.batch) * p.h_kv * N, D) ||
      !make_tmap(&mv, v, uint64_t(p.batch) * p.h_kv * N, D))
    return cudaErrorInvalidValue;
  auto kern = attn_tc_kernel<D, BLK, TOKEN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::SMEM);
  if (e != cudaSuccess) return e;
  const unsigned grid = unsigned(p.batch) * p.h_q * ((p.seqlen + BM - 1) / BM);
  kern<<<grid, kThreads, Cfg<D>::SMEM, st>>>(mq, mk, mv, tile_idx, tile_cnt, static_cast<__nv_bfloat16*>(o),
                                             lse, p, ws, wait_limit);
  return cudaGetLastError();
}

}  // namespace

cudaError_t run_attention(const crisp_params& p, const void* q, const void* k, const void* v,
                          const int32_t* tile_idx, const int32_t* tile_cnt, void* o, float* lse,
                          void* ws, cudaStream_t st, long long wait_limit) {
  // token-granular lists carry per-tile flags (block 128 only, checked by the ABI)
  const bool token = tile_idx && p.vs_granularity == CRISP_GRAN_TOKEN && p.block == 128;
  const long long wl = wait_limit;
  if (p.head_dim == 64) {
    if (token) return launch_tc<64, 128, true>(p, q, k, v, tile_idx, tile_cnt, o, lse, ws, st, wl);
    return p.block == 64 ? launch_tc<64, 64, false>(p, q, k, v, tile_idx, tile_cnt, o, lse, ws, st, wl)
                         : launch_tc<64, 128, false>(p, q, k, v, tile_idx, tile_cnt, o, lse, ws, st, wl);
  }
  if (token) return launch_tc<128, 128, true>(p, q, k, v, tile_idx, tile_cnt, o, lse, ws, st, wl);
  return p.block == 64 ? launch_tc<128, 64, false>(p, q, k, v, tile_idx, tile_cnt, o, lse, ws, st, wl)
                       : launch_tc<128, 128, false>(p, q, k, v, tile_idx, tile_cnt, o, lse, ws, st, wl);
}

}  // namespace crisp
