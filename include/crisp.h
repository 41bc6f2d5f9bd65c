/*
 * crisp.h — C ABI of the B200 (sm_100a) CRISP sparse-prefill library.
 *
 * The operation is CRISP sparse attention prefill as defined by the paper
 * "CRISP: Cliff-awaRe Input-adaptive Sparse Prefilling with
 * Structural-Mass-Motivated Routing": Algorithm 1 (route each head, select a
 * sparse index set, attend over it), with PatSearch (Algorithm 2), the
 * sink-aware VS index (Algorithm 3, Eq. 3-4), the PE index (Algorithm 4),
 * the FlexPrefill JSD router and gamma VS index kept as comparison paths
 * (Appendix A, Algorithms 5-6) and block-sparse attention (Eq. 1).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors q, k, v, o are DEVICE pointers to contiguous bf16 arrays of
 *    layout [batch][heads][seqlen][head_dim] (heads = h_q for q and o,
 *    h_kv for k and v). GQA: query head h reads KV head h / (h_q / h_kv).
 *    Every pointer must be 16-byte aligned.
 *  - The caller owns all memory, including the workspace `ws` of
 *    `ws_bytes` >= crisp_workspace_size(p) bytes (256-byte aligned). The
 *    library allocates no device memory and keeps no global state, except
 *    the fixed scratch array of crisp_route_noalloc (see there).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream). The return value covers argument validation and
 *    launch errors only; kernel-side errors (a bounded wait that ran out,
 *    an out-of-range tile index or sequence length) are recorded in a status
 *    word held in the first 8 bytes of `ws`, read back (and cleared) with
 *    crisp_get_device_status(). crisp_route and crisp_dense_prefill start a
 *    prefill and clear the word (crisp_route also clears the per-head
 *    completion counters its kernels keep right after it); a caller who runs
 *    crisp_select or crisp_sparse_prefill alone on a new workspace zeroes
 *    those 8 bytes.
 *  - Block geometry: N_b = ceil(n / block) for a sequence of n tokens
 *    (CRISP paper, Section 4.3); the last block may be partial. block is 64
 *    or 128; head_dim is 64 or 128; with N_b = ceil(seqlen / block),
 *    3 <= N_b <= 8192 and ceil(N_b / 64) <= block; batch * h_q <= 65535 and
 *    batch * h_q * seqlen < 2^31 (rows of q addressed by 32-bit tile
 *    coordinates). Anything else returns CRISP_ERR_SHAPE.
 *  - Variable lengths: with p->seq_lens == NULL every sequence has seqlen
 *    tokens. Otherwise seq_lens is a DEVICE array of batch int32 lengths
 *    and sequence b occupies the first seq_lens[b] rows of its
 *    [seqlen][head_dim] slices; the other rows are padding that no result
 *    depends on. Each length must satisfy 2*block < n <= seqlen (N_b >= 3);
 *    a kernel that meets one outside clamps it into that range and records
 *    CRISP_ERR_DEVICE. Padding rows of v must hold finite values up to the
 *    next multiple of 128 rows (the tensor cores multiply them by exact
 *    zeros; zeros are the natural filler). Per-block outputs beyond a
 *    sequence's own N_b are zero (p_v, p_s, tile_cnt, mask, vs_sel); rows
 *    of o beyond its length are zero and their lse is -inf.
 *  - Return codes: CRISP_OK, or a negative crisp_status. Invalid arguments
 *    never launch a kernel.
 */
#ifndef CRISP_H_
#define CRISP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CRISP_OK = 0,
  CRISP_ERR_ARG = -1,        /* null pointer, misaligned pointer, bad enum or hyper-parameter */
  CRISP_ERR_SHAPE = -2,      /* unsupported or inconsistent shape */
  CRISP_ERR_WORKSPACE = -3,  /* workspace smaller than crisp_workspace_size() */
  CRISP_ERR_CUDA = -4,       /* a CUDA runtime call or kernel launch failed */
  CRISP_ERR_TIMEOUT = -5,    /* device status: a bounded wait inside a kernel ran out */
  CRISP_ERR_DEVICE = -6      /* device status: a kernel found an out-of-range index */
} crisp_status;

typedef enum { CRISP_ROUTER_CSTRUCT = 0, CRISP_ROUTER_JSD = 1 } crisp_router;
/* VS selection rule: ALPHA = Algorithm 3 with the mean floor of Eq. 3;
 * GAMMA = Algorithm 6 (Appendix A); ALPHA_MEDIAN = Algorithm 3 with the
 * median floor of Appendix H (Table 9). */
typedef enum { CRISP_VS_ALPHA = 0, CRISP_VS_GAMMA = 1, CRISP_VS_ALPHA_MEDIAN = 2 } crisp_vs_rule;
typedef enum { CRISP_PATTERN_VS = 0, CRISP_PATTERN_PE = 1 } crisp_pattern;
/* Granularity of a VS head's mask in Eq. 1: TILE executes the selected
 * vertical and slash blocks as whole tiles (the default); TOKEN keeps whole
 * tiles for vertical blocks but lets a slash block admit only the key-query
 * pairs on its diagonal band (slash index j + n-1-t in the block). TOKEN
 * requires block 128. */
typedef enum { CRISP_GRAN_TILE = 0, CRISP_GRAN_TOKEN = 1 } crisp_granularity;

/* Problem and hyper-parameters (CRISP paper, Section 5 Setup: tau_proxy 0.2,
 * gamma 0.95 for PE, alpha 1.0, block 128, k_min 8 blocks per direction). */
typedef struct {
  int32_t batch, h_q, h_kv, seqlen, head_dim, block;
  float alpha;         /* noise-floor multiplier of Eq. 4 (> 0) */
  float gamma;         /* cumulative coverage of Algorithms 4 and 6, in (0, 1] */
  float tau_proxy;     /* C_struct routing threshold of Algorithm 2 */
  float tau_jsd;       /* JSD routing threshold of Algorithm 5 (not given by the paper) */
  int32_t k_min_blocks;/* minimum blocks per VS direction (k_min of Algorithm 3), >= 1 */
  int32_t router;      /* crisp_router */
  int32_t vs_rule;     /* crisp_vs_rule */
  float sm_scale;      /* softmax scale; 0 selects 1/sqrt(head_dim) */
  int32_t vs_granularity;  /* crisp_granularity */
  const int32_t* seq_lens; /* device [batch] sequence lengths, or NULL (all = seqlen) */
} crisp_params;

/* Library version (major*10000 + minor*100 + patch). */
int crisp_version(void);

/* Human-readable name of a crisp_status value (static string). */
const char* crisp_status_string(int status);

/* Validates `p` without launching anything. Returns CRISP_OK or the error. */
int crisp_check_params(const crisp_params* p);

/* Workspace bytes needed by route, select and the prefill kernels for `p`
 * (0 when `p` is invalid). One workspace may serve all calls of a prefill
 * issued in order on one stream. */
size_t crisp_workspace_size(const crisp_params* p);

/* Stage (a)+(b) of Algorithm 1: PatSearch (Algorithm 2) for every head.
 * Computes the causal proxy map of the last `block` query rows against all
 * keys without materialising it, its block scores
 *   p_v[b][h][N_b]  (vertical: per-key mean over proxy rows, block sums),
 *   p_s[b][h][N_b]  (slash: per-diagonal means, block sums; diagonal of
 *                    entry (r, j) indexed by j + block - 1 - r),
 * and routes each head: pattern[b*h_q+h] = CRISP_PATTERN_VS iff
 *   C_struct = p_v[0] + p_v[N_b-1] >= tau_proxy      (router CSTRUCT, Eq. 2)
 *   D_JS(p_v, pooled estimate) >= tau_jsd              (router JSD, Algorithm 5).
 * score[b*h_q+h] receives C_struct or D_JS. All outputs are device arrays
 * (pattern int32, the rest float32); none may be NULL. */
int crisp_route(const crisp_params* p, const void* q, const void* k, void* ws, size_t ws_bytes,
                int32_t* pattern, float* score, float* p_v, float* p_s, void* stream);

/* Stage (c): index selection and tile lists.
 * VS heads: per direction, Algorithm 3 (vs_rule ALPHA: blocks with
 * p > alpha*mu, mu = max(1-p[0]-p[N_b-1],0)/(N_b-2), count clipped to
 * [k_min, N_b], top-k by score, ties to the lower block; vs_rule
 * ALPHA_MEDIAN: the same with mu = the median of p[1..N_b-2], the mean of
 * the two middle values for an even count) or Algorithm 6
 * (vs_rule GAMMA: smallest prefix of the descending scores reaching gamma,
 * clipped the same way); the union with vertical block 0 and slash block
 * N_b-1 marks tile (qb, kb <= qb) iff kb is a selected vertical block or
 * the tile holds a causal (t, j) pair whose slash index j + n-1-t falls in a
 * selected slash block: for n a multiple of block, iff qb-kb or qb-kb-1 is
 * a selected slash offset (offset = N_b-1-slash id); for a partial last
 * block a slash block can meet three tile diagonals.
 * PE heads: Algorithm 4 — block-mean pooling of Q and K, causal block
 * softmax, entries divided by N_b, smallest descending prefix reaching
 * gamma (ties to the lower flat id qb*N_b+kb), plus tiles (qb,qb), (qb,0).
 * Outputs (device): tile_cnt[b][h][N_b] (int32) and tile_idx[b][h][N_b][N_b]
 * (int32; row (b,h,qb) holds tile_cnt ascending key-block ids, the rest
 * undefined; with CRISP_GRAN_TOKEN each entry also carries flags above bit
 * 24: bit 24 = whole tile (vertical block, block 0 or a PE head), bits
 * 25..27 = slash blocks N_b-1-delta+e selected for e = -1, 0, +1, with
 * delta = qb - kb; the key-block id is entry & 0xFFFFFF); mask[b][h][N_b][N_b] (uint8 0/1, upper triangle 0) unless
 * mask == NULL; vs_sel[b][h][2][N_b] (uint8 0/1: selected vertical, then
 * slash blocks; all 0 for PE heads) unless vs_sel == NULL.
 * pattern, p_v, p_s are crisp_route's outputs. */
int crisp_select(const crisp_params* p, const void* q, const void* k, const int32_t* pattern,
                 const float* p_v, const float* p_s, void* ws, size_t ws_bytes, uint8_t* mask,
                 uint8_t* vs_sel, int32_t* tile_idx, int32_t* tile_cnt, void* stream);

/* Stage (d): causal GQA block-sparse attention, Eq. 1, over the tiles
 * listed by crisp_select (whole tiles; token-level causal mask inside).
 * o: bf16 [b][h_q][seqlen][head_dim]. lse (may be NULL): float32
 * [b][h_q][seqlen], natural-log sum of exp of the scaled logits. */
int crisp_sparse_prefill(const crisp_params* p, const void* q, const void* k, const void* v,
                         const int32_t* tile_idx, const int32_t* tile_cnt, void* o, float* lse,
                         void* ws, size_t ws_bytes, void* stream);

/* Dense causal attention with the same kernel over every causal tile (the
 * paper's exact-attention baseline, Section 5). Same layouts as above. */
int crisp_dense_prefill(const crisp_params* p, const void* q, const void* k, const void* v,
                        void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/* Device workspace bytes crisp_prefill_host needs for `p` with
 * `kv_per_chunk` KV heads per chunk (0 when the arguments are invalid). */
size_t crisp_prefill_host_workspace_size(const crisp_params* p, int kv_per_chunk);

/* Algorithm 1 end to end on HOST buffers: route (Algorithm 2), select
 * (Algorithms 3, 4, 6) and block-sparse attention (Eq. 1), exactly as
 * crisp_route + crisp_select + crisp_sparse_prefill, for inputs and outputs
 * in page-locked host memory (cudaHostAlloc / cudaMallocHost or
 * cudaHostRegister over the whole array).
 *  - q, k, v: host bf16 [batch][heads][seqlen][head_dim]; o: host bf16
 *    [batch][h_q][seqlen][head_dim]; lse (may be NULL): host float32
 *    [batch][h_q][seqlen]. Only the first seq_lens[b] rows of sequence b are
 *    read and written; other rows of o and lse keep their contents.
 *  - seq_lens (may be NULL = all seqlen): HOST int32 [batch], each in
 *    (2*block, seqlen] (else CRISP_ERR_SHAPE). p->seq_lens must be NULL.
 *  - pattern (may be NULL): host int32 [batch * h_q] receiving the routes.
 *  - The prefill runs in chunks of one sequence and kv_per_chunk KV heads
 *    (a divisor of h_kv) with their query heads. Two slots of device
 *    buffers in `ws` (caller-owned device memory, 256-byte aligned, at least
 *    crisp_prefill_host_workspace_size bytes) alternate between chunks: the
 *    host-to-device copies of chunk i+1 and the device-to-host copies of
 *    chunk i-1 overlap the kernels of chunk i (one cudaMemcpy2DAsync per
 *    tensor and chunk). The kernels run on `stream`, after the work already
 *    queued there; the copies on two streams the call creates and destroys.
 *  - The call is synchronous: it returns once o (and lse, pattern) hold the
 *    result. Kernel-side errors of any chunk are returned directly
 *    (CRISP_ERR_TIMEOUT, CRISP_ERR_DEVICE); pageable host pointers return
 *    CRISP_ERR_ARG before any copy. The library allocates no device memory. */
int crisp_prefill_host(const crisp_params* p, const void* q, const void* k, const void* v, void* o,
                       float* lse, const int32_t* seq_lens, int32_t* pattern, int kv_per_chunk,
                       void* ws, size_t ws_bytes, void* stream);

/* Routing without a caller workspace. The paper has no counterpart: this
 * entry point exists for callers that may not allocate device memory — for
 * example a plug-in whose host framework reserves all device memory for its
 * own pool and passes no workspace, or a latency-critical loop that cannot
 * take the device-wide synchronisation cudaMalloc may cause. It runs exactly
 * the crisp_route kernels, with identical arguments and outputs minus the
 * workspace, and calls no allocator. Its scratch is one fixed array of
 * CRISP_NOALLOC_SCRATCH_BYTES in the library's device image, held by every
 * GPU that loads the library until the process exits.
 *  - Problems whose routing scratch exceeds that size (Llama shapes beyond
 *    32k tokens, for instance) return CRISP_ERR_WORKSPACE without launching.
 *  - All calls on a device share the array, which keeps the last call's
 *    contents; calls whose kernels overlap on the GPU race. Issue them in
 *    order on one stream.
 *  - Each call outside stream capture looks up the array's address (with
 *    the device current); during capture the address of the last lookup on
 *    that device is used, so make the first call on a device before any
 *    stream capture.
 *  - Kernel-side errors (a bounded wait that ran out, an out-of-range entry
 *    of seq_lens) are recorded in a status word at the start of the array;
 *    read and clear it with crisp_get_device_status(NULL, ...). */
#define CRISP_NOALLOC_SCRATCH_BYTES (16u << 20)
int crisp_route_noalloc(const crisp_params* p, const void* q, const void* k, int32_t* pattern,
                        float* score, float* p_v, float* p_s, void* stream);

/* Diagnostic: exercises the bounded wait that every pipelined kernel of the
 * library uses (on an mbarrier phase, a TMA copy or a tensor-core commit).
 * One CTA waits on an mbarrier nothing arrives on, gives up after
 * `limit_cycles` (1 .. 2^31) SM clock cycles, records CRISP_ERR_TIMEOUT in
 * the status word of `ws` (256-byte aligned, at least 256 bytes; read it with
 * crisp_get_device_status) and returns; the context stays usable. Returns
 * CRISP_ERR_ARG for a bad workspace or limit. The paper has no counterpart. */
int crisp_selftest_wait_timeout(void* ws, long long limit_cycles, void* stream);

/* Diagnostic: runs the two pipelined tensor-core kernels of a prefill — the
 * proxy statistics kernel of crisp_route and the attention kernel of
 * crisp_dense_prefill — on the given problem with every pipeline wait cut to
 * `limit_cycles` (1 .. 2^20 - 1) SM clock cycles, short enough that waits run
 * out. A CTA whose wait runs out records CRISP_ERR_TIMEOUT in the status word
 * of `ws`, leaves its loops, waits (bounded) for the copies and tensor-core
 * operations it has in flight, releases its tensor memory and returns; the
 * context stays usable and the next call of any entry point runs normally.
 * `o` and the routing scratch of `ws` hold unspecified values afterwards.
 * Arguments as for crisp_dense_prefill (validated the same way; a limit out
 * of range returns CRISP_ERR_ARG). The paper has no counterpart. */
int crisp_selftest_pipeline_timeout(const crisp_params* p, const void* q, const void* k, const void* v,
                                    void* o, void* ws, size_t ws_bytes, long long limit_cycles,
                                    void* stream);

/* Synchronises `stream`, copies the device status word out of `ws` into
 * *status (CRISP_OK or CRISP_ERR_TIMEOUT / CRISP_ERR_DEVICE) and clears it.
 * ws == NULL reads the status word of crisp_route_noalloc's scratch array on
 * the current device. Returns CRISP_OK unless the copy itself failed
 * (CRISP_ERR_CUDA) or status is NULL / ws misaligned (CRISP_ERR_ARG). */
int crisp_get_device_status(void* ws, int32_t* status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CRISP_H_ */
