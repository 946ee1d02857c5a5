/*
 * mla.h -- C ABI of the B200 (sm_100a) Multi-head Latent Attention hot path.
 *
 * What is computed (DeepSeek-V2, "DeepSeek-V2 summary" (7shi.hateblo.jp),
 * App. C "Full Formulas of MLA" and §2.1.2-§2.1.3):
 *
 *   c^Q_t  = W_DQ h_t          q^C_t = W_UQ c^Q_t        q^R_t = RoPE(W_QR c^Q_t)
 *   c^KV_t = W_DKV h_t         k^R_t = RoPE(W_KR h_t)   (shared by all heads)
 *   o_{t,i} = sum_{j<=t} softmax_j([q^C;q^R]_{t,i} . [W_UK_i c^KV_j ; k^R_j] / sqrt(d_h+d_R)) W_UV_i c^KV_j
 *   u_t    = W_O [o_{t,1}; ...; o_{t,n_h}]
 *
 * Only [c^KV_t | k^R_t] (d_c + d_R elements per token) is cached (App. C,
 * the boxed vectors; §2.1.4).  Decode uses the absorbed form from the last
 * paragraph of App. C: W_UK is folded into the query and W_UV is applied to
 * the latent output, so per-head keys and values are never formed.  Prefill
 * forms them once per token (the un-absorbed form) because there every key
 * serves many queries.
 *
 * Conventions shared by every entry point
 *  - Weights use the pages' shapes W in R^{out x in} (y = W x), row-major,
 *    dtype `mla_dims.dtype`.  Head i owns rows [i d_h, (i+1) d_h) of W_UQ,
 *    W_UK, W_UV, rows [i d_R, (i+1) d_R) of W_QR and columns
 *    [i d_h, (i+1) d_h) of W_O.  Shapes: W_DQ [d_cq x d], W_UQ [n_h d_h x q_in],
 *    W_QR [n_h d_R x q_in] with q_in = d_cq (or d when d_cq == 0), W_DKV
 *    [d_c x d], W_KR [d_R x d], W_UK and W_UV [n_h d_h x d_c], W_O [d x n_h d_h].
 *  - RoPE rotates interleaved pairs (2m, 2m+1) by pos * rope_base^(-2m/d_R);
 *    pos is the token's 0-based index in its sequence.
 *  - Cache row of a token: [c^KV (d_c) | RoPE'd k^R (d_R)], dtype
 *    `mla_dims.dtype`, row stride (d_c + d_R) elements (or the E4M3 row of
 *    `mla_cache_format`), contiguous per sequence (token p of sequence s in
 *    row seq_start[s] + p) or paged through a block table.
 *  - All pointers except the structs themselves are device pointers owned by
 *    the caller.  The library allocates nothing and keeps no state between
 *    calls (apart from the diagnostic timing hook at the end of this file).
 *    Work is enqueued on `stream` and the calls return without synchronising.
 *  - Every device pointer must be 16-byte aligned (TMA requirement).
 *  - Supported shapes.  bf16 storage runs on the tensor-core kernels, which
 *    are built for the DeepSeek-V2 head shape: d_h = 128, d_R = 64,
 *    d_c = 512, n_h <= 128, d_model and d_cq multiples of 64 (this covers
 *    DeepSeek-V2 and DeepSeek-V2-Lite).  fp32 storage runs on CUDA-core
 *    kernels for small layers: d_c <= 512 (a multiple of 4), d_h <= 256,
 *    d_R even, 16-byte rows.  Anything else returns MLA_ERR_UNSUPPORTED
 *    with nothing enqueued; no call switches to another kernel family.
 *  - Errors in arguments, shapes, alignment or workspace size are found on the
 *    host and returned before anything is enqueued.  Faults found on the
 *    device set bits of a status word in the workspace, which
 *    `mla_get_device_status` reads: 1 = a cache write at a position at or
 *    beyond `capacity` (or outside the cache) was skipped; 2 = a pipeline
 *    wait timed out; 4 = the decode planner saw a negative seqlen; 8 = the
 *    decode attention met scores of a sequence that rose, within one run of
 *    64-token tiles, more than 96 (in units of log2, after the softmax
 *    scale) above the maximum of the tiles before them, which is past the
 *    kernel's range (that sequence's u is not valid).
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mla_stream_t;   /* same type as cudaStream_t; NULL = legacy default stream */

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = -1,   /* NULL pointer, non-positive size, inconsistent dims */
    MLA_ERR_UNSUPPORTED = -2,   /* dims/dtype outside what the kernels implement */
    MLA_ERR_MISALIGNED = -3,    /* a device pointer is not 16-byte aligned */
    MLA_ERR_WORKSPACE = -4,     /* workspace NULL or smaller than mla_workspace_bytes() */
    MLA_ERR_CUDA = -5,          /* a CUDA runtime/driver call failed (launch, tensor map) */
    MLA_ERR_DEVICE_FAULT = -6   /* a kernel reported a fault through the status word */
} mla_status;

typedef enum { MLA_BF16 = 0, MLA_FP32 = 1 } mla_dtype;

typedef struct {
    int d_model;       /* d: hidden size */
    int n_h;           /* attention heads */
    int d_h;           /* per-head dimension of q^C, k^C, v */
    int d_R;           /* per-head rotary dimension (d_e on some pages), even */
    int d_c;           /* KV compression dimension (latent width) */
    int d_cq;          /* query compression dimension d_c'; 0 = no query compression (V2-Lite) */
    double rope_base;  /* RoPE base, e.g. 10000 */
    int dtype;         /* mla_dtype: storage type of h, weights and cache */
    /* YaRN context extension (DeepSeek-V2 summary §3.1.4): 0 = off (plain
     * RoPE, softmax scale 1/sqrt(d_h+d_R)).  With yarn_s >= 1 the rotary pairs
     * of q^R and k^R use the YaRN frequencies: pair m keeps
     * theta_m = rope_base^(-2m/d_R) when yarn_L0 (the pre-training length)
     * spans more than yarn_beta of its wavelengths 2 pi / theta_m, takes
     * theta_m / yarn_s below yarn_alpha of them and blends linearly in
     * between; every attention score is multiplied by t with
     * sqrt(t) = 0.0707 ln(yarn_s) + 1.  The pages give s = 40, alpha = 1,
     * beta = 32 and a 4K pre-training length.  Requires yarn_beta > yarn_alpha
     * >= 0 and yarn_L0 > 0. */
    double yarn_s, yarn_alpha, yarn_beta, yarn_L0;
    /* mla_cache_format of the latent cache (0 = storage dtype rows). */
    int cache_format;
} mla_dims;

/* Latent cache row formats.
 *  MLA_CACHE_DTYPE: [c^KV (d_c) | k^R (d_R)] in the storage dtype; row stride
 *    (d_c + d_R) elements.
 *  MLA_CACHE_E4M3: the low-bit cache of DeepSeek-V2 summary §3.2.3 (about 6
 *    bits per element there; FP8 here, the serving example's format family):
 *    bytes [0, d_c) c^KV as OCP E4M3 codes, [d_c, d_c + 2 d_R) k^R in bf16,
 *    byte d_c + 2 d_R the row's scale exponent k (int8), then zeros to
 *    d_c + 2 d_R + 16 (the row stride, 656 bytes at DeepSeek-V2 dims against
 *    1152 for bf16).  Element j of c^KV is code_value * 2^k, with k the
 *    smallest integer for which max_j |c^KV_j| / 2^k <= 448 (the largest E4M3
 *    value; k = 0 for an all-zero row), and the code the E4M3 value nearest
 *    to c^KV_j / 2^k, ties to even.  bf16 storage only; mla_prefill does not
 *    take it (MLA_ERR_UNSUPPORTED) — fill such a cache with mla_cache_append
 *    and mla_decode. */
typedef enum { MLA_CACHE_DTYPE = 0, MLA_CACHE_E4M3 = 1 } mla_cache_format;

typedef struct {
    const void* W_DQ;  /* [d_cq x d]; ignored when d_cq == 0 */
    const void* W_UQ;
    const void* W_QR;
    const void* W_DKV;
    const void* W_UK;
    const void* W_UV;
    const void* W_KR;
    const void* W_O;
    /* RMSNorm gains of the compressed latents (DeepSeek-V2 summary §3.1.2,
     * which adds RMSNorm layers after them; App. C has none).  NULL = no norm.
     * g_kv [d_c]: c^KV is normalised, x / sqrt(mean(x^2) + 1e-6) * g_kv, before
     * it is cached.  g_q [d_cq]: c^Q is normalised the same way before the
     * up-projections (only with query compression: g_q with d_cq == 0 is
     * MLA_ERR_INVALID_ARG).  Storage dtype, 16-byte aligned. */
    const void* g_kv;
    const void* g_q;
} mla_weights;

typedef struct {
    void* base;                 /* device: rows of (d_c + d_R) elements */
    const int64_t* seq_start;   /* device [n_seq]: row of token 0 of each sequence (contiguous
                                   layout; unused, may be NULL, when block_table is given) */
    const int32_t* capacity;    /* device [n_seq] or NULL: rows reserved per sequence; a write at
                                   pos >= capacity[s] is skipped and raises MLA_ERR_DEVICE_FAULT */
    int64_t n_rows;             /* rows allocated at `base` (> 0): bounds of every tile load; a
                                   write at a row >= n_rows is skipped and raises MLA_ERR_DEVICE_FAULT */
    /* Paged layout (optional; NULL = contiguous per sequence).  The cache is a
     * pool of pages of block_size rows (a multiple of 64); token p of sequence
     * s lives in row block_table[s * max_blocks + p / block_size] * block_size
     * + p % block_size.  device int32 [n_seq x max_blocks], caller-owned.  A
     * position p >= max_blocks * block_size is treated as beyond capacity. */
    const int32_t* block_table;
    int32_t block_size;
    int32_t max_blocks;
} mla_cache;

/* Bytes of workspace needed by mla_decode for batches up to `max_batch` and by
 * mla_cache_append / mla_prefill for up to `max_tokens` tokens per call.  The
 * workspace is caller-owned device memory (256-byte aligned); one workspace
 * must not be used by two calls that run at the same time.  Its first 256
 * bytes hold the device status word: zero them once when the workspace is
 * created (mla_get_device_status clears the word after reading a fault).  The
 * rest may hold anything; the calls never read what they did not write. */
size_t mla_workspace_bytes(const mla_dims* dims, int max_batch, int max_tokens);

/* Cache append (the cache-write half of App. C): for t in [0, T),
 *   row = seq_start[seq_idx[t]] + pos[t]
 *   cache[row] = [ c^KV = W_DKV h_t | k^R = RoPE_{pos[t]}(W_KR h_t) ]  rounded to the cache dtype.
 * h: device [T x d_model]; seq_idx, pos: device int32 [T]. */
mla_status mla_cache_append(const mla_dims* dims, const mla_weights* w,
                            const void* h, int T,
                            const int32_t* seq_idx, const int32_t* pos,
                            const mla_cache* cache,
                            void* workspace, size_t workspace_bytes,
                            mla_stream_t stream);

/* Decode step (App. C with absorption): one new token per sequence b in [0, B).
 * seqlen[b] (device int32) = L_b tokens already cached for sequence b.  The new
 * token's cache row is written at position L_b (row seq_start[b] + L_b) and the
 * token attends over positions 0..L_b.  seqlen is not modified.
 * h: device [B x d_model]; u: device fp32 [B x d_model] (output, overwritten). */
mla_status mla_decode(const mla_dims* dims, const mla_weights* w,
                      const void* h, int B,
                      const mla_cache* cache, const int32_t* seqlen,
                      float* u,
                      void* workspace, size_t workspace_bytes,
                      mla_stream_t stream);

/* Causal prefill of T tokens of sequence `seq` at positions start_pos .. start_pos+T-1
 * (App. C with j <= t).  Writes their cache rows, then each token attends over
 * the cached prefix (positions < start_pos, already in the cache) and over the
 * new tokens up to itself.  h: device [T x d_model]; u: device fp32 [T x d_model]. */
mla_status mla_prefill(const mla_dims* dims, const mla_weights* w,
                       const void* h, int T, int start_pos,
                       const mla_cache* cache, int seq,
                       float* u,
                       void* workspace, size_t workspace_bytes,
                       mla_stream_t stream);

/* Synchronises `stream`, reads and clears the device status word kept in the
 * workspace.  Returns MLA_OK, MLA_ERR_DEVICE_FAULT (a kernel flagged a fault;
 * *detail, if non-NULL, receives the fault bits) or MLA_ERR_CUDA. */
mla_status mla_get_device_status(void* workspace, mla_stream_t stream, int* detail);

/* Static description of a status code. */
const char* mla_status_string(mla_status s);

/* Byte offset inside the workspace of an intermediate left by the last
 * mla_decode call with batch `max_batch` (ids 0-4) or by the last
 * mla_cache_append / mla_prefill call of up to `max_tokens` tokens (id 5),
 * for inspection in tests.  0-4 are in the storage dtype: 0 = c^Q [B x d_cq],
 * 1 = q^C [B x n_h d_h], 2 = Q_lat [B x n_h x (d_c+d_R)] = [W_UK_i^T q^C_i ; q^R_i]
 * pre-multiplied by log2(e)/sqrt(d_h+d_R), 3 = O_lat [B x n_h x d_c]
 * (normalised latent output), 4 = o [B x n_h d_h].  5 = c^KV of the tokens
 * in fp32 [T x d_c] as the down-projection produced it, before the RMSNorm
 * and the E4M3 encoding (written only when one of them is on).  Returns
 * (size_t)-1 for an unknown id or invalid dims. */
size_t mla_workspace_offset(const mla_dims* dims, int max_batch, int max_tokens, int which);

/* ---------------------------------------------------------------------------
 * Decode step that allocates nothing.  No counterpart in the paper: this is a
 * deployment convenience around mla_decode.
 *
 * Some callers cannot allocate device memory when they call into this library,
 * so they cannot hand it a workspace: for example an engine plugin that is given
 * only its input and output buffers, or a latency-critical path where cudaMalloc
 * (which can synchronise the whole device) is not allowed.  This entry point
 * takes the same arguments as mla_decode minus the workspace and computes the
 * same u.  Its scratch is one file-scope __device__ array of
 * MLA_STATIC_SCRATCH_BYTES that every GPU which loads this library holds until
 * the process exits; the call itself allocates nothing (no cudaMalloc, no
 * cudaFree, no allocating library routine).
 *
 *  - Limit: the decode scratch of batch B must fit in the array.  At
 *    DeepSeek-V2 dims it is about 0.35 MB x B (per-token intermediates)
 *    + 0.26 MB x (B + SMs/2) (attention partials) + 0.15 MB x (split-K tile
 *    width, 32..256), so B up to 101 on a 148-SM B200; V2-Lite dims allow far
 *    larger batches.  A batch that does not fit returns MLA_ERR_WORKSPACE with
 *    nothing enqueued.
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current) and keeps it for the life of the
 *    process.  Make that first call outside any stream capture, and do not
 *    reset the device (cudaDeviceReset) between calls: the kept address
 *    would no longer be mapped.
 *  - All calls share the one array, and it keeps the previous call's contents;
 *    each call clears what must start at zero.  Calls whose work overlaps on the
 *    GPU (several streams or host threads) race on the array.
 *  - Faults found on the device are not reported (there is no workspace for
 *    mla_get_device_status); the variant's status word is cleared at each call.
 */
#define MLA_STATIC_SCRATCH_BYTES (96u << 20)
mla_status mla_decode_static(const mla_dims* dims, const mla_weights* w,
                             const void* h, int B,
                             const mla_cache* cache, const int32_t* seqlen,
                             float* u, mla_stream_t stream);

/* Diagnostic: exercises the bounded pipeline waits every kernel uses.  Runs a
 * one-thread-block kernel whose wait on a shared-memory barrier is never
 * satisfied; after the time limit (2 s) the wait gives up, sets
 * FAULT_WAIT_TIMEOUT (2) in the workspace's status word and the kernel exits,
 * leaving the context usable.  Read the result with mla_get_device_status.
 * workspace: as for the other calls (256-byte aligned, status word zeroed). */
mla_status mla_check_wait_timeout(void* workspace, mla_stream_t stream);

/* Diagnostic: number of kernels this library has launched in this process
 * (all entry points, all threads).  The difference across a call counts the
 * call's kernel launches. */
unsigned long long mla_kernel_launches(void);

/* Diagnostic timing hook.  While set, every mla_decode / mla_prefill call
 * records CUDA event `begin` (a cudaEvent_t) on its stream just before the
 * launch of its attention kernel and `end` just after it, so a caller can time
 * that kernel alone.  NULL, NULL clears it.  Process-wide setting; callers on
 * several threads must not use it concurrently. */
void mla_set_attention_events(void* begin, void* end);

#ifdef __cplusplus
}
#endif
#endif /* MLA_B200_H */
