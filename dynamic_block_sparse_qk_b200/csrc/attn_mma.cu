// Block-sparse causal GQA flash attention (CRISP paper, Eq. 1) on the legacy
// warp-level tensor-core path (mma.sync m16n8k16, bf16 -> fp32).
//
// CTA = 4 warps = 64 query rows; key steps of 64 keys; K/V tiles double
// buffered in XOR-swizzled shared memory with cp.async; online softmax in
// the exp2 domain. A listed key block of width `block` is visited as
// block/64 key steps; steps wholly above the causal diagonal are skipped.
#include "common.cuh"
#include "kernels.h"

namespace crisp {

template <int D>
__global__ void __launch_bounds__(128, 2) attn_mma_kernel(const __nv_bfloat16* __restrict__ q,
                                                          const __nv_bfloat16* __restrict__ k,
                                                          const __nv_bfloat16* __restrict__ v,
                                                          const int32_t* __restrict__ tile_idx,
                                                          const int32_t* __restrict__ tile_cnt,
                                                          __nv_bfloat16* __restrict__ o,
                                                          float* __restrict__ lse, crisp_params p,
                                                          void* ws) {
  constexpr int BM = 64, BN = 64;
  constexpr int ROWB = D * 2, CPR = D / 8;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* qs = smem;                         // [BM][D]
  unsigned char* ks = qs + BM * ROWB;               // [2][BN][D]
  unsigned char* vs = ks + 2 * BN * ROWB;           // [2][BN][D]
  const Workspace W = make_workspace(p);
  int32_t* status = ws_ptr<int32_t>(ws, W.status);

  const int nslab = p.seqlen / BM;
  const int slab = nslab - 1 - int(blockIdx.x);     // heavy (late) slabs first
  const int bh = blockIdx.y;
  const int b = bh / p.h_q, h = bh % p.h_q, hk = h / (p.h_q / p.h_kv);
  const int nb = p.seqlen / p.block;
  const int qb = slab * BM / p.block;
  const int sub_per = p.block / BN;
  const size_t N = size_t(p.seqlen);
  const int row0 = slab * BM;
  const __nv_bfloat16* qh = q + (size_t(bh) * N + row0) * D;
  const __nv_bfloat16* kh = k + (size_t(b) * p.h_kv + hk) * N * D;
  const __nv_bfloat16* vh = v + (size_t(b) * p.h_kv + hk) * N * D;
  const int32_t* list = tile_idx ? tile_idx + (size_t(bh) * nb + qb) * nb : nullptr;
  int cnt = tile_idx ? tile_cnt[size_t(bh) * nb + qb] : qb + 1;
  if (cnt < 0 || cnt > qb + 1) {     // a list longer than the causal row cannot be valid
    if (threadIdx.x == 0) report_error(status, CRISP_ERR_DEVICE, cnt);
    cnt = cnt < 0 ? 0 : qb + 1;
  }
  const int nsteps = cnt * sub_per;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const float sl2 = (p.sm_scale > 0.f ? p.sm_scale : rsqrtf(float(D))) * kLog2e;

  // key start of step s, or -1 when the step is skipped
  auto step_key0 = [&](int s) -> int {
    const int i = s / sub_per, sub = s % sub_per;
    int kb = list ? list[i] : i;
    if (kb < 0 || kb > qb) {
      report_error(status, CRISP_ERR_DEVICE, kb);
      return -1;
    }
    const int key0 = kb * p.block + sub * BN;
    return key0 > row0 + BM - 1 ? -1 : key0;
  };
  auto load_rows = [&](unsigned char* dst, const __nv_bfloat16* src, int rows) {
    const uint32_t base = smem_u32(dst);
    for (int i = tid; i < rows * CPR; i += 128) {
      const int row = i / CPR, c = i % CPR;
      cp_async16(base + swz(row, c, ROWB), src + size_t(row) * D + c * 8);
    }
  };

  load_rows(qs, qh, BM);
  int next = 0, key_next = -1;
  while (next < nsteps && (key_next = step_key0(next)) < 0) ++next;
  if (key_next >= 0) {
    load_rows(ks, kh + size_t(key_next) * D, BN);
    load_rows(vs, vh + size_t(key_next) * D, BN);
  }
  cp_async_commit();

  uint32_t qf[D / 16][4];
  float oacc[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const int rA = row0 + warp * 16 + g;   // this thread's rows: rA, rA + 8

  int buf = 0, it = 0;
  while (key_next >= 0) {
    const int key0 = key_next;
    // find and prefetch the following step
    ++next;
    key_next = -1;
    while (next < nsteps && (key_next = step_key0(next)) < 0) ++next;
    cp_async_wait<0>();
    __syncthreads();
    if (key_next >= 0) {
      load_rows(ks + (buf ^ 1) * BN * ROWB, kh + size_t(key_next) * D, BN);
      load_rows(vs + (buf ^ 1) * BN * ROWB, vh + size_t(key_next) * D, BN);
    }
    cp_async_commit();
    if (it == 0) {
      const uint32_t qbase = smem_u32(qs);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        ldmatrix_x4(qbase + swz(warp * 16 + (lane & 15), kk * 2 + (lane >> 4), ROWB), qf[kk][0],
                    qf[kk][1], qf[kk][2], qf[kk][3]);
    }
    // S = Q K^T (16 x 64 per warp)
    float s[BN / 8][4];
#pragma unroll
    for (int j = 0; j < BN / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
    const uint32_t kbase = smem_u32(ks + buf * BN * ROWB);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int j = 0; j < BN / 8; j += 2) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(kbase + swz(j * 8 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1), ROWB),
                    b0, b1, b2, b3);
        mma_bf16_16816(s[j], qf[kk], b0, b1);
        mma_bf16_16816(s[j + 1], qf[kk], b2, b3);
      }
    }
    const bool diag = key0 + BN - 1 > row0 + warp * 16;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = rA + half * 8;
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < BN / 8; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float x = s[j][half * 2 + e] * sl2;
          if (diag && key0 + j * 8 + t4 * 2 + e > row) x = -INFINITY;
          s[j][half * 2 + e] = x;
          mx = fmaxf(mx, x);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(mrow[half], mx);
      const float corr = fast_exp2(mrow[half] - mnew);
      mrow[half] = mnew;
      float ls = 0.f;
#pragma unroll
      for (int j = 0; j < BN / 8; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float pe = fast_exp2(s[j][half * 2 + e] - mnew);
          s[j][half * 2 + e] = pe;
          ls += pe;
        }
      lrow[half] = lrow[half] * corr + ls;   // per-thread partial; reduced at the end
#pragma unroll
      for (int j = 0; j < D / 8; ++j) {
        oacc[j][half * 2] *= corr;
        oacc[j][half * 2 + 1] *= corr;
      }
    }
    // O += P V
    const uint32_t vbase = smem_u32(vs + buf * BN * ROWB);
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int j = 0; j < D / 8; j += 2) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(vbase + swz(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), j + (lane >> 4), ROWB),
                          b0, b1, b2, b3);
        mma_bf16_16816(oacc[j], a, b0, b1);
        mma_bf16_16816(oacc[j + 1], a, b2, b3);
      }
    }
    buf ^= 1;
    ++it;
  }
  cp_async_wait<0>();
  // epilogue
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float l = lrow[half];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int row = rA + half * 8;
    __nv_bfloat16* orow = o + (size_t(bh) * N + row) * D;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      *reinterpret_cast<uint32_t*>(orow + j * 8 + t4 * 2) =
          pack_bf16(oacc[j][half * 2] * inv, oacc[j][half * 2 + 1] * inv);
    }
    if (lse && t4 == 0) lse[size_t(bh) * N + row] = (mrow[half] + log2f(l)) * kLn2;
  }
}

cudaError_t run_attention(const crisp_params& p, const void* q, const void* k, const void* v,
                          const int32_t* tile_idx, const int32_t* tile_cnt, void* o, float* lse,
                          void* ws, cudaStream_t st) {
  dim3 grid(p.seqlen / 64, p.batch * p.h_q);
  if (p.head_dim == 64) {
    const size_t smem = size_t(5) * 64 * 64 * 2;
    attn_mma_kernel<64><<<grid, 128, smem, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), tile_idx, tile_cnt, static_cast<__nv_bfloat16*>(o), lse, p, ws);
  } else {
    const size_t smem = size_t(5) * 64 * 128 * 2;
    cudaFuncSetAttribute(attn_mma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    attn_mma_kernel<128><<<grid, 128, smem, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), tile_idx, tile_cnt, static_cast<__nv_bfloat16*>(o), lse, p, ws);
  }
  return cudaGetLastError();
}

}  // namespace crisp
