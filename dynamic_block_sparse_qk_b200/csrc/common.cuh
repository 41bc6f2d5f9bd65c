// Shared device helpers and the workspace layout of the CRISP sm_100a library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/crisp.h"

namespace crisp {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxBlocks = 8192;  // N_b limit (selection kernels keep one row in smem)

// ----------------------------------------------------------------------------
// Workspace layout. Every region is 256-byte aligned. The caller allocates
// `total` bytes once per problem shape; all stages share it in stream order.
// ----------------------------------------------------------------------------
struct Workspace {
  size_t status;      // int32[64]: [0] status word, [1] first bad index
  size_t head_cnt;    // uint32[BH][4]: per-head CTA completion counters (proxy, histogram, ties; one spare)
  size_t stat_m;      // float[BH][Nb][R]   per-row max of a proxy key tile (log2 units)
  size_t stat_lo;     // float[BH][Nb][R]   sum exp2(s-m) over tile columns c <= r
  size_t stat_hi;     // float[BH][Nb][R]   sum exp2(s-m) over tile columns c >  r
  size_t chunk_m;     // float[BH][NC][R]   per-row max over a chunk of key tiles (NC = ceil(Nb / proxy_chunk))
  size_t chunk_l;     // float[BH][NC][R]   per-row sum over the chunk (scaled to chunk_m)
  size_t row_m;       // float[BH][R]       proxy row max
  size_t row_l;       // float[BH][R]       proxy row normaliser
  size_t kbar;        // float[B*Hkv][Nb][d] block means of K
  size_t qbar;        // float[BH][Nb][d]    block means of Q (PE heads)
  size_t sel;         // uint8[BH][2][Nb]    selected vertical / slash blocks
  size_t sel_bits;    // uint32[BH][2][ceil(Nb/32)] the same as bitmasks, plus vertical 0 / slash Nb-1
  size_t abar;        // float[BH][Nb][Nb]   PE estimate divided by N_b
  size_t hist_cnt;    // uint32[BH][4096]    radix-select bucket counts
  size_t hist_sum;    // double[BH][4096]    radix-select bucket sums
  size_t pe_state;    // PeState[BH]
  size_t eq_cnt;      // uint32[BH][Nb]      per-row count of entries equal to the cut value
  size_t total;
};

struct PeState {
  uint32_t prefix;     // decided high bits of the cut value
  uint32_t all;        // 1 when the whole triangle sums below gamma (select all)
  uint32_t m_equal;    // how many entries equal to the cut value are taken
  uint32_t pad;
  double above_sum;    // sum of entries strictly above the decided range
};

// Blocks of the longest sequence: N_b = ceil(seqlen / block) (the storage
// stride of every per-block array).
__host__ __device__ inline int n_blocks(const crisp_params& p) { return (p.seqlen + p.block - 1) / p.block; }

// Length of sequence b: seq_lens[b] clamped to (2 * block, seqlen], or
// seqlen without a length array. `status` (may be NULL) records a length
// outside that range as CRISP_ERR_DEVICE.
__device__ inline void report_error(int32_t* status, int32_t code, int32_t where);
__device__ inline int seq_len(const crisp_params& p, int b, int32_t* status = nullptr) {
  if (!p.seq_lens) return p.seqlen;
  const int n = p.seq_lens[b];
  const int lo = 2 * p.block + 1;
  if (n < lo || n > p.seqlen) {
    if (status) report_error(status, CRISP_ERR_DEVICE, n);
    return n < lo ? lo : p.seqlen;
  }
  return n;
}

// Key tiles per proxy CTA: small enough that short sequences still give about
// four CTAs per SM (148 SMs), at most 32 for long ones; even, so a 128-key
// step of 64-wide blocks never straddles two chunks.
__host__ __device__ inline int proxy_chunk(const crisp_params& p) {
  const long long nb = n_blocks(p);
  long long c = (nb * p.batch * p.h_q + 591) / 592;
  c = c < 4 ? 4 : (c > 32 ? 32 : c);
  return int((c + 1) & ~1ll);
}

enum HeadCounter { kCntProxy = 0, kCntHist = 1, kCntEq = 2 };   // slot 3 spare

// Tile-list entries in token granularity: key-block id in the low 24 bits,
// then flags (whole tile; slash blocks N_b-1-delta-1, N_b-1-delta, N_b-delta).
constexpr int32_t kTileIdMask = 0xFFFFFF;
constexpr int32_t kTileWhole = 1 << 24;
constexpr int kTileSlashShift = 25;

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline Workspace make_workspace(const crisp_params& p) {
  Workspace w{};
  const size_t BH = size_t(p.batch) * p.h_q;
  const size_t BK = size_t(p.batch) * p.h_kv;
  const size_t nb = size_t(n_blocks(p));
  const size_t R = size_t(p.block);
  const size_t nc = (nb + proxy_chunk(p) - 1) / proxy_chunk(p);
  const size_t d = size_t(p.head_dim);
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  w.status = take(64 * 4);
  w.head_cnt = take(BH * 4 * 4);
  w.stat_m = take(BH * nb * R * 4);
  w.stat_lo = take(BH * nb * R * 4);
  w.stat_hi = take(BH * nb * R * 4);
  w.chunk_m = take(BH * nc * R * 4);
  w.chunk_l = take(BH * nc * R * 4);
  w.row_m = take(BH * R * 4);
  w.row_l = take(BH * R * 4);
  w.kbar = take(BK * nb * d * 4);
  w.qbar = take(BH * nb * d * 4);
  w.sel = take(BH * 2 * nb);
  w.sel_bits = take(BH * 2 * ((nb + 31) / 32) * 4);
  w.abar = take(BH * nb * nb * 4);
  w.hist_cnt = take(BH * 4096 * 4);
  w.hist_sum = take(BH * 4096 * 8);
  w.pe_state = take(BH * sizeof(PeState));
  w.eq_cnt = take(BH * nb * 4);
  w.total = off;
  return w;
}

// Bytes at the start of the workspace that a routing call clears: the status
// word and the per-head completion counters (adjacent regions).
inline size_t route_clear_bytes(const crisp_params& p) {
  const Workspace w = make_workspace(p);
  return w.head_cnt + size_t(p.batch) * p.h_q * 4 * 4;
}

template <typename T>
__host__ __device__ inline T* ws_ptr(void* base, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<char*>(base) + off);
}

// Records the first device-side error in the status word (index kept for debugging).
__device__ inline void report_error(int32_t* status, int32_t code, int32_t where) {
  if (atomicCAS(status, 0, code) == 0) status[1] = where;
}

// ----------------------------------------------------------------------------
// Warp-level helpers.
// ----------------------------------------------------------------------------
__device__ inline float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ inline float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ inline double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ inline float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ inline uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ inline uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace crisp
