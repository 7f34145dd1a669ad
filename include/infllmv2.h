/*
 * infllmv2.h -- C ABI of the B200 (sm_100a) InfLLM v2 block-sparse attention library.
 *
 * InfLLM v2 splits the KV cache into fixed-size blocks, represents every block by
 * "semantic kernels" (compressed keys), lets every query token pick its most relevant
 * blocks (one set shared by all query heads of a GQA group) and runs exact attention
 * over the picked blocks only.  Sources:
 *   "MiniCPM4：端设备上的超高效大型语言模型" (MiniCPM4 summary page), s2.1.1 (block units,
 *   per-token top blocks), s2.1.2 (relevance via semantic kernels, group-shared
 *   selection), s2.1.3 (attention only with the most relevant blocks);
 *   "OpenBMB publishes Minicpm4 ..." news page, "Technical innovations in MinicPM4"
 *   (semantic kernels, dynamic block selection for prefill and decode).
 * The block/kernel sizes, the pooling rules and the forced blocks come from the
 * workload definition (block 64, kernel 32 stride 16, mean-pooled kernels,
 * kernel-to-block max-pool, group-sum, top-k including 1 initial + 2 local blocks).
 *
 * Conventions for every entry point
 *  - Tensors are device pointers, row-major with the innermost index last, and must
 *    be 16-byte aligned.  bf16 means IEEE bfloat16 bit patterns (uint16_t storage).
 *  - The caller allocates and owns every buffer.  The library allocates nothing,
 *    keeps no per-call state, and may be called concurrently on distinct streams.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Host-side argument checks run before anything is launched: on a
 *    negative status nothing was launched and no output was touched.
 *  - A kernel that waits on the GPU never waits without a bound: if an internal wait
 *    exceeds its limit the kernel stops early and sets a device error word, which
 *    infllmv2_device_error() reads.  The word is sticky: until its wait-timeout bit
 *    is cleared, later waits give up at once, so outputs of that call and of later
 *    calls are undefined.
 *  - Query positions: prefill queries are tokens 0..L-1 of a fresh sequence; a chunk's
 *    queries are the last q_lens[b] tokens of a cache of kv_lens[b] tokens; a decode
 *    query is the last token of its sequence, at position lens[b]-1.  A query's own key
 *    and value are always in the cache.
 *  - GQA: q-head h uses kv-head h / (num_q_heads / num_kv_heads).
 */
#ifndef INFLLMV2_H_
#define INFLLMV2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define INFLLMV2_API __attribute__((visibility("default")))
#else
#define INFLLMV2_API
#endif

/* Same type as cudaStream_t, without requiring the CUDA headers. */
typedef struct CUstream_st* infllmv2_stream_t;

/* Status codes (return value of every entry point). */
enum {
  INFLLMV2_OK = 0,
  INFLLMV2_ERR_INVALID_ARG = -1,   /* null / misaligned pointer, bad size or count */
  INFLLMV2_ERR_UNSUPPORTED = -2,   /* valid but not implemented (e.g. head_dim != 128) */
  INFLLMV2_ERR_WORKSPACE = -3,     /* workspace missing or smaller than required */
  INFLLMV2_ERR_CUDA = -4           /* a CUDA runtime call or kernel launch failed */
};

/* Device error word bits (infllmv2_device_error). */
enum {
  INFLLMV2_DEVERR_WAIT_TIMEOUT = 1, /* an internal wait ran out of its time limit */
  INFLLMV2_DEVERR_CACHE_FULL = 2    /* infllmv2_append_kv met lens[b] outside [0, Lmax) */
};

enum { INFLLMV2_MODE_PREFILL = 0, INFLLMV2_MODE_DECODE = 1 };

/* Operations for infllmv2_workspace_size. */
enum {
  INFLLMV2_OP_COMPRESS = 0,
  INFLLMV2_OP_SELECT_PREFILL = 1,
  INFLLMV2_OP_SELECT_DECODE = 2,
  INFLLMV2_OP_ATTN_PREFILL = 3,
  INFLLMV2_OP_ATTN_DECODE = 4,
  INFLLMV2_OP_ATTN_BACKWARD = 5
};

/* Problem description shared by all calls.
 *   batch          B >= 1
 *   num_q_heads    Hq, a multiple of num_kv_heads; Hq / Hkv must be 1, 2, 4, 8 or 16
 *   num_kv_heads   Hkv >= 1
 *   head_dim       d; only 128 is implemented
 *   block_size     KV block length in tokens; only 64 is implemented
 *   kernel_size    semantic-kernel length; only 32 is implemented
 *   kernel_stride  distance between kernel starts; only 16 is implemented
 *   topk           blocks per (query token, kv-head), forced ones included; 1..256
 *   n_init         initial blocks always selected (blocks 0..n_init-1), >= 0
 *   n_local        local blocks always selected (the query's block and the
 *                  n_local-1 blocks before it), >= 0; n_init + n_local <= topk
 *   softmax_scale  scale of q.k in scoring and attention; <= 0 means 1/sqrt(d)
 *   score_mode     block score (INFLLMV2_SCORE_*); 0 = softmax-sum
 *   pool_mode      kernel-to-block pooling (INFLLMV2_POOL_*); 0 = overlapping kernels
 * A zero-initialised struct with the sizes filled in selects the default reading.    */
typedef struct {
  int32_t batch, num_q_heads, num_kv_heads, head_dim;
  int32_t block_size, kernel_size, kernel_stride;
  int32_t topk, n_init, n_local;
  float softmax_scale;
  int32_t score_mode, pool_mode;
} infllmv2_params;

/* Variants of the block score and of the pooling ([S] s2.1.2 names the relevance score
 * through fine-grained semantic kernels without a formula; s2.1.3 lists hyper-parameter
 * choices without values).  With m_h(j) the max scaled logit of head h over the
 * kernels pooled into block j:
 *   INFLLMV2_SCORE_SOFTMAX_SUM  S(j) = sum_h exp(m_h(j) - lse_h), lse_h over every visible
 *                               kernel (two passes over the kernels)
 *   INFLLMV2_SCORE_LOGIT_SUM    S(j) = sum_h m_h(j) (one pass, no lse; may be negative)
 *   INFLLMV2_POOL_OVERLAP       block j pools every kernel overlapping it (4j-1 .. 4j+3)
 *   INFLLMV2_POOL_INSIDE        block j pools the kernels inside it (4j .. 4j+2); a block
 *                               is eligible once kernel 4j is visible                  */
enum { INFLLMV2_SCORE_SOFTMAX_SUM = 0, INFLLMV2_SCORE_LOGIT_SUM = 1 };
enum { INFLLMV2_POOL_OVERLAP = 0, INFLLMV2_POOL_INSIDE = 1 };

/* Largest sequence length (prefill L or decode Lmax) the kernels accept. */
#define INFLLMV2_MAX_SEQ_LEN 262144

/* Number of semantic kernels in n tokens: (n - kernel_size) / kernel_stride + 1 when
 * n >= kernel_size, else 0. */
INFLLMV2_API int64_t infllmv2_num_kernels(const infllmv2_params* p, int64_t n);

/* Key compression into semantic kernels ([S] s2.1.2; "semantic kernels" of the news
 * page).  Kernel i of (b, g) is the mean of key rows [16 i, 16 i + 32), computed exactly
 * (fp64 sums) and rounded once to bf16 (nearest even).
 *   k     bf16 [B, Hkv, Lmax, d]   (input)
 *   lens  int32 [B] device, or NULL: sequence b holds lens[b] <= Lmax tokens; with
 *         NULL every sequence holds Lmax tokens.  Kernels past NK(lens[b]) are not
 *         written.
 *   kc    bf16 [B, Hkv, NK(Lmax), d]   (output; may be NULL when NK(Lmax) == 0)
 * Returns INVALID_ARG for null/misaligned pointers or Lmax outside
 * [1, INFLLMV2_MAX_SEQ_LEN]. */
INFLLMV2_API int infllmv2_compress_keys(const infllmv2_params* p, const void* k, const int32_t* lens,
                           int32_t Lmax, void* kc, infllmv2_stream_t stream);

/* Group-shared top-k block selection ([S] s2.1.1, s2.1.2).  For every (b, kv-head g,
 * query token at position t):
 *   x_h(i) = scale * q_h . Kc_i  for the group's heads h and the kernels i whose last
 *            token is <= t;
 *   lse_h  = log sum_i exp(x_h(i));
 *   m_h(j) = max of x_h(i) over the visible kernels overlapping block j (kernels
 *            4j-1 .. 4j+3; with INFLLMV2_POOL_INSIDE, 4j .. 4j+2);
 *   S(j)   = sum over the group's heads of exp(m_h(j) - lse_h) (with
 *            INFLLMV2_SCORE_LOGIT_SUM, of m_h(j)).
 * Forced blocks (0..n_init-1 and cur-n_local+1..cur, cur = t / 64) are always taken;
 * the other topk - |forced| slots go to the eligible blocks with the highest S, lower
 * block index first on equal S.  Each row of block_idx is written ascending and
 * padded with -1.
 *   mode       INFLLMV2_MODE_PREFILL: q bf16 [B, L, Hq, d], lens must be NULL,
 *              L_or_Lmax = L, kc from infllmv2_compress_keys over L tokens,
 *              block_idx int32 [B, Hkv, L, topk].
 *              INFLLMV2_MODE_DECODE: q bf16 [B, Hq, d], lens int32 [B] device
 *              (1 <= lens[b] <= Lmax), L_or_Lmax = Lmax, kc [B, Hkv, NK(Lmax), d],
 *              block_idx int32 [B, Hkv, 1, topk].
 *   ws, ws_bytes  device workspace of at least infllmv2_workspace_size(p,
 *              INFLLMV2_OP_SELECT_PREFILL or _DECODE, L_or_Lmax) bytes (may be NULL
 *              when that size is 0, which it is for both modes in this version).
 *              Contents on entry do not matter.
 *  Decode runs one thread-block cluster of up to 16 CTAs per (b, g); a device that
 *  cannot co-schedule that cluster gets INFLLMV2_ERR_UNSUPPORTED before any launch. */
INFLLMV2_API int infllmv2_select_blocks(const infllmv2_params* p, int mode, const void* q, const void* kc,
                           const int32_t* lens, int32_t L_or_Lmax, int32_t* block_idx,
                           void* ws, size_t ws_bytes, infllmv2_stream_t stream);

/* Sparse attention for prefill ([S] s2.1.3).  For every (b, token t, q-head h):
 *   O = softmax(scale * q . K_J^T) V_J over the keys J of the selected blocks of
 *   (b, h / G, t), cut at position t (causal inside the query's own block).
 *   q          bf16 [B, L, Hq, d];  k, v  bf16 [B, Hkv, L, d]
 *   block_idx  int32 [B, Hkv, L, topk], ascending or not, unique entries, -1 = unused;
 *              entries outside [0, t / 64] are skipped.
 *   o          bf16 [B, L, Hq, d] (output)
 *   lse        fp32 [B, Hq, L] natural-log normaliser (output), or NULL. */
INFLLMV2_API int infllmv2_sparse_attn_prefill(const infllmv2_params* p, const void* q, const void* k,
                                 const void* v, const int32_t* block_idx, int32_t L, void* o,
                                 float* lse, void* ws, size_t ws_bytes, infllmv2_stream_t stream);

/* Chunked / ragged-batch prefill: a chunk of queries against an existing cache ([S] s2.1:
 * prefill of long contexts; s2.1.1-s2.1.2: every query token selects its own blocks;
 * news page "Technical innovations in MinicPM4": dynamic context block selection).
 * Sequence b's cache holds kv_lens[b] tokens (its keys, values and semantic kernels,
 * e.g. from earlier chunks), and its chunk is the last q_lens[b] of them: query row r
 * sits at position kv_lens[b] - q_lens[b] + r.  The selection and attention are those
 * of infllmv2_select_blocks / infllmv2_sparse_attn_prefill at those positions; a fresh
 * prefill is the case q_lens = kv_lens = NULL, Lq = Lmax = L.
 *   q          bf16 [B, Lq, Hq, d]: rows 0..q_lens[b]-1 of sequence b are its chunk,
 *              rows at or past q_lens[b] are padding
 *   q_lens     int32 [B] device, or NULL (every chunk holds Lq queries)
 *   kv_lens    int32 [B] device, or NULL (every cache holds Lmax tokens); values are
 *              clamped on the GPU to kv_lens[b] in [0, Lmax], q_lens[b] in
 *              [0, min(Lq, kv_lens[b])]
 *   Lq, Lmax   1 <= Lq <= Lmax <= INFLLMV2_MAX_SEQ_LEN
 *   kc         bf16 [B, Hkv, NK(Lmax), d] (infllmv2_compress_keys with lens = kv_lens)
 *   block_idx  int32 [B, Hkv, Lq, topk] (output of the selection, input of the attention)
 *   k, v       bf16 [B, Hkv, Lmax, d]
 *   o          bf16 [B, Lq, Hq, d];  lse fp32 [B, Hq, Lq] or NULL
 * Padding rows (r >= q_lens[b]) of block_idx, o and lse are not written.  No workspace
 * (ws may be NULL).  INVALID_ARG for null / misaligned pointers or sizes out of range. */
INFLLMV2_API int infllmv2_select_blocks_chunk(const infllmv2_params* p, const void* q, int32_t Lq, const void* kc,
                                              const int32_t* q_lens, const int32_t* kv_lens, int32_t Lmax,
                                              int32_t* block_idx, void* ws, size_t ws_bytes,
                                              infllmv2_stream_t stream);
INFLLMV2_API int infllmv2_sparse_attn_chunk(const infllmv2_params* p, const void* q, int32_t Lq, const void* k,
                                            const void* v, const int32_t* q_lens, const int32_t* kv_lens,
                                            int32_t Lmax, const int32_t* block_idx, void* o, float* lse, void* ws,
                                            size_t ws_bytes, infllmv2_stream_t stream);

/* Sparse attention for one decode token per sequence ([S] s2.1.3, prefill *and*
 * decode per s2.1 of the same page).  Split over the selected blocks across CTAs,
 * then merged with the partial log-sum-exps: inside a thread-block cluster per
 * (b, kv-head) (no workspace) when B * Hkv >= SMs / 16, else through the workspace.
 *   q          bf16 [B, Hq, d];  k_cache, v_cache bf16 [B, Hkv, Lmax, d]
 *   lens       int32 [B] device, 1 <= lens[b] <= Lmax; the query sits at lens[b]-1
 *   block_idx  int32 [B, Hkv, 1, topk] (as for prefill)
 *   o          bf16 [B, Hq, d];  lse fp32 [B, Hq] or NULL
 *   ws         at least infllmv2_workspace_size(p, INFLLMV2_OP_ATTN_DECODE, Lmax) bytes;
 *              may be NULL when that size is 0 */
INFLLMV2_API int infllmv2_sparse_attn_decode(const infllmv2_params* p, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* lens, int32_t Lmax,
                                const int32_t* block_idx, void* o, float* lse, void* ws,
                                size_t ws_bytes, infllmv2_stream_t stream);

/* One whole decode step in one launch: optionally the cache maintenance of
 * infllmv2_append_kv for the new token, then infllmv2_select_blocks(DECODE) and
 * infllmv2_sparse_attn_decode on the list it selects ([S] s2.1: the block selection
 * serves decoding as well as prefill; s2.1.2: the group's heads share the blocks and the
 * semantic kernels summarise the cached keys; s2.1.3: attention over the selected blocks
 * only).  A thread-block cluster per (b, kv-head) scores Kc, selects the blocks and
 * attends to them without a round trip through global memory, so clusters overlap each
 * other's selection and attention.  Same results as the separate calls: block_idx
 * bit-identical, o and lse from the same per-block arithmetic (the split of the list over
 * the cluster's CTAs may differ, so o and lse may differ from the separate call in the
 * last bits).
 *   q          bf16 [B, Hq, d]
 *   k_new, v_new  bf16 [B, Hkv, d], or both NULL.  Given: lens[b] counts the cached
 *              tokens before the step; the token's rows are written at position lens[b]
 *              of the caches and the semantic kernel it completes to kc (exactly as
 *              infllmv2_append_kv), the query sits at lens[b] and lens_out[b] = lens[b] + 1.
 *              A sequence with lens[b] outside [0, Lmax) is not appended (lens_out[b] =
 *              lens[b], INFLLMV2_DEVERR_CACHE_FULL in the device error word).  NULL: the
 *              caches already hold the query's token, which sits at min(lens[b], Lmax) - 1.
 *   k_cache, v_cache  bf16 [B, Hkv, Lmax, d] (written only when appending)
 *   kc         bf16 [B, Hkv, NK(Lmax), d] (may be NULL when NK(Lmax) = 0 and nothing is appended)
 *   lens       int32 [B] device (read only); a sequence with no query (length <= 0) gets
 *              an all -1 list, o = 0 and lse = -inf
 *   lens_out   int32 [B] device, distinct from lens; required when appending, else ignored
 *   block_idx  int32 [B, Hkv, 1, topk] (output)
 *   o          bf16 [B, Hq, d];  lse fp32 [B, Hq] or NULL
 * No workspace.  INVALID_ARG for null / misaligned pointers (or k_new without v_new,
 * lens_out missing or equal to lens), UNSUPPORTED when the device cannot hold one cluster
 * of the chosen size. */
INFLLMV2_API int infllmv2_decode_step(const infllmv2_params* p, const void* q, const void* k_new, const void* v_new,
                                      void* k_cache, void* v_cache, void* kc, const int32_t* lens, int32_t* lens_out,
                                      int32_t Lmax, int32_t* block_idx, void* o, float* lse,
                                      infllmv2_stream_t stream);

/* Backward of the prefill sparse attention over fixed block lists ([S] s2.1, s2.1.3:
 * the sparse attention is trained; the top-k block choice is constant almost
 * everywhere, so the gradients reach q, k and v through the attention only and the block
 * lists are inputs).  With P = softmax(scale q K_J^T) over the keys J of a row's blocks
 * cut at its position t, D = sum_d dO O:
 *   dq = scale sum_u P_u (dO.V_u - D) K_u,  dK_u += scale P_u (dO.V_u - D) q,
 *   dV_u += P_u dO.
 *   q, o, d_o  bf16 [B, L, Hq, d] (o and lse from infllmv2_sparse_attn_prefill on the
 *              same inputs; P is recomputed from lse)
 *   k, v       bf16 [B, Hkv, L, d];  lse fp32 [B, Hq, L]
 *   block_idx  int32 [B, Hkv, L, topk] as for the forward (unique entries per row)
 *   dq         bf16 [B, L, Hq, d];  dk, dv bf16 [B, Hkv, L, d] (outputs)
 *   ws         at least infllmv2_workspace_size(p, INFLLMV2_OP_ATTN_BACKWARD, L) bytes
 *              (contents on entry do not matter; about 8 bytes x (topk / 2 + 2 d) per
 *              (token, kv-head)).
 * dq is deterministic; dk and dv are summed over a block's query rows by several CTAs
 * with fp32 atomics, so their rounding may differ between runs.  Fresh sequences only
 * (query t at position t).  WORKSPACE for a missing or short workspace, INVALID_ARG for
 * null / misaligned pointers. */
INFLLMV2_API int infllmv2_sparse_attn_backward(const infllmv2_params* p, const void* q, const void* k,
                                               const void* v, const void* o, const float* lse, const void* d_o,
                                               const int32_t* block_idx, int32_t L, void* dq, void* dk, void* dv,
                                               void* ws, size_t ws_bytes, infllmv2_stream_t stream);

/* Decode sparse attention that allocates nothing and takes no workspace.  The paper has
 * no counterpart to this entry point: it exists for callers that cannot allocate device
 * memory at call time -- e.g. an engine plugin whose execute step must not allocate, or
 * a service that reserves its whole memory budget at start-up and forbids later
 * cudaMalloc.  Same arguments and results as infllmv2_sparse_attn_decode without
 * ws/ws_bytes; when the problem takes the workspace path (few sequences), the split
 * partials live in a fixed 8 MiB array inside the library
 * (INFLLMV2_NOALLOC_SCRATCH_BYTES), which every GPU that loads the library holds until
 * the process exits.
 *  - Returns INFLLMV2_ERR_WORKSPACE, without launching anything, when the problem needs
 *    more scratch than that (the need is infllmv2_workspace_size(p,
 *    INFLLMV2_OP_ATTN_DECODE, Lmax)).  With the split rule of this version the need
 *    stays below about 2.5 MB for every valid parameter set, so the check is a guard
 *    against future split rules rather than a limit callers meet.
 *  - The first call on a device looks up the array's device address (one
 *    cudaGetSymbolAddress, with that device current); make that first call before any
 *    stream capture.
 *  - Every call on a device uses the same array, and nothing in it needs to start at
 *    zero (each call overwrites the parts it reads).  Two calls whose kernels overlap on
 *    the GPU (e.g. on two streams) race on the array and give undefined results: order
 *    them on one stream or with events. */
#define INFLLMV2_NOALLOC_SCRATCH_BYTES (8u << 20)
INFLLMV2_API int infllmv2_sparse_attn_decode_noalloc(const infllmv2_params* p, const void* q,
                                                     const void* k_cache, const void* v_cache,
                                                     const int32_t* lens, int32_t Lmax,
                                                     const int32_t* block_idx, void* o, float* lse,
                                                     infllmv2_stream_t stream);

/* Decode cache maintenance: appends one token per sequence ([S] s2.1: decoding; s2.1.2:
 * the semantic kernels summarise the cached keys).  For every b and kv-head g the new
 * key and value rows are written at position lens[b] of the caches; when the new length
 * n = lens[b] + 1 completes a semantic kernel (n >= 32 and (n - 32) % 16 == 0), kernel
 * i = (n - 32) / 16, the mean of key rows [16 i, 16 i + 32), is written to kc -- the value
 * infllmv2_compress_keys gives for the same cache; then lens[b] = n.  The caller runs it
 * once per decode step, before infllmv2_select_blocks, on the same stream.
 *   k_new, v_new      bf16 [B, Hkv, d]
 *   k_cache, v_cache  bf16 [B, Hkv, Lmax, d] (updated in place)
 *   lens              int32 [B] device (in: cached tokens; out: + 1)
 *   kc                bf16 [B, Hkv, NK(Lmax), d] (updated in place)
 * A sequence with lens[b] outside [0, Lmax) is left untouched and sets
 * INFLLMV2_DEVERR_CACHE_FULL in the device error word (checked on the GPU: lens lives
 * there).  No workspace. */
INFLLMV2_API int infllmv2_append_kv(const infllmv2_params* p, const void* k_new, const void* v_new, void* k_cache,
                                    void* v_cache, int32_t* lens, int32_t Lmax, void* kc,
                                    infllmv2_stream_t stream);

/* Workspace bytes needed by `op` (INFLLMV2_OP_*) for sequence length L_or_Lmax, or 0
 * when the op needs none; (size_t)-1 for invalid parameters. */
INFLLMV2_API size_t infllmv2_workspace_size(const infllmv2_params* p, int op, int32_t L_or_Lmax);

/* Validates a parameter block; returns INFLLMV2_OK or the status a call would get. */
INFLLMV2_API int infllmv2_check_params(const infllmv2_params* p);

/* Static text for a status code. */
INFLLMV2_API const char* infllmv2_status_string(int status);

/* Reads (and, if clear != 0, resets) the device error word of the current device.
 * Synchronises the device.  Returns the INFLLMV2_DEVERR_* bits, or a negative status. */
INFLLMV2_API int infllmv2_device_error(int clear);

/* Library version, as major * 10000 + minor * 100 + patch. */
INFLLMV2_API int infllmv2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* INFLLMV2_H_ */
