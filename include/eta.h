/*
 * eta.h — C ABI of libeta.so: B200 (sm_100a) block-sparse decode attention for
 * Elastic Threshold Attention (ETA).
 *
 * Method: "Elastic Threshold Attention: Learned Contextual Sparsity for
 * Long-Context Decoding" (Haris, Li, Karimzadehgan). Section references below
 * are to the picx.dev summary of that paper (Methodology §1-§4, Eq. 1-5) and
 * to the figure captions on the thelatestinai.com page (Figure 1, Figure 6).
 *
 * Conventions shared by every entry point
 *  - Every pointer argument is DEVICE memory owned by the caller, unless the
 *    argument says "host". The library keeps no allocation of its own; the
 *    per-call scratch lives in a caller-provided workspace.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and returns after enqueueing its kernels. Calls
 *    on distinct streams with distinct workspaces may run concurrently.
 *  - Arguments are validated on the host before anything is launched; a
 *    rejected call returns ETA_ERR_INVALID_ARG / ETA_ERR_UNSUPPORTED /
 *    ETA_ERR_WORKSPACE and enqueues nothing. A failed launch returns
 *    ETA_ERR_CUDA. Errors detected on the device (a bounded wait that ran
 *    out) are recorded in the workspace status word: read them with
 *    eta_read_device_status.
 *  - Layouts (row-major, innermost last):
 *      q      [B][Hq][d]          kv_dtype-independent: q_dtype
 *      K, V   [B][Hkv][capacity][d]  kv_dtype; token s of (b, kv head h) at
 *                                 ((b*Hkv + h)*capacity + s)*d
 *      meta   mu, var [B][Hkv][d][nb_cap] fp32 (coordinate-major, so one warp
 *             lane per block reads coalesced), maxnorm [B][Hkv][nb_cap] fp32,
 *             nb_cap = capacity / block_size
 *      tau    thresholds indexed tau[b*tau_batch_stride + h]; a stride of 0
 *             broadcasts one per-head constant over the batch
 *      out    [B][Hq][d] fp32
 *  - n_tokens counts the cached tokens INCLUDING the current one (the cache is
 *    appended before attention); the current token is t = n_tokens - 1. Query
 *    head h reads kv head h / (Hq / Hkv) (grouped-query attention).
 */
#ifndef ETA_H_
#define ETA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ETA_ABI_VERSION 3

#if defined(__GNUC__)
#define ETA_API __attribute__((visibility("default")))
#else
#define ETA_API
#endif

typedef struct CUstream_st* eta_stream_t; /* same type as cudaStream_t */

typedef enum {
  ETA_OK = 0,
  ETA_ERR_INVALID_ARG = 1,    /* a null pointer, bad size, misaligned pointer */
  ETA_ERR_UNSUPPORTED = 2,    /* a shape the library has no kernel for */
  ETA_ERR_WORKSPACE = 3,      /* workspace null, misaligned or too small */
  ETA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
  ETA_ERR_DEVICE_TIMEOUT = 5  /* a device-side wait exceeded its limit */
} eta_status_t;

/* ETA_FP8_E4M3: one byte per element, 1 sign, 4 exponent (bias 7) and 3
 * mantissa bits, no infinities (the "fn" variant: S.1111.111 is NaN, 448 the
 * largest value). K and V only; every stored value widens exactly. */
typedef enum { ETA_F32 = 0, ETA_BF16 = 1, ETA_FP8_E4M3 = 2 } eta_dtype_t;

/* Problem shape. Supported: head_dim in {64, 128}; block_size in
 * {16, 32, 64, 128}; n_q_heads a multiple of n_kv_heads with group size
 * Hq/Hkv in {1, 2, 4, 8}; capacity a positive multiple of block_size;
 * capacity / block_size < 2^24; q_dtype ETA_F32 or ETA_BF16; kv_dtype
 * ETA_F32, ETA_BF16 or ETA_FP8_E4M3 (the last with a bf16 q and head_dim 128;
 * ETA_ERR_UNSUPPORTED otherwise). */
typedef struct {
  int32_t batch;        /* B */
  int32_t n_q_heads;    /* Hq */
  int32_t n_kv_heads;   /* Hkv */
  int32_t head_dim;     /* d (d_h) */
  int32_t block_size;   /* b: tokens per KV block (Methodology §4) */
  int64_t capacity;     /* tokens allocated per (batch, kv head) */
  int32_t kv_dtype;     /* eta_dtype_t of K and V */
  int32_t q_dtype;      /* eta_dtype_t of q */
} eta_shape_t;

/* Method parameters. */
typedef struct {
  float beta;          /* gate temperature of Eq. 2 (the end of its anneal, 5.0) */
  float z;             /* screening confidence z of Eq. 5 */
  float offset_a;      /* threshold offset a: the screen compares with tau - a */
  int32_t n_local;     /* trailing blocks admitted without screening (>= 1; the
                          last block holds the current token, whose gate Eq. 3
                          exempts) */
  int32_t n_splits;    /* decode work ranges (thread blocks); 0 = one per SM */
  int32_t gate;        /* ETA_GATE_SIGMOID (Eq. 2-3) or ETA_GATE_HARD (strict mode) */
  int32_t sub_blocks;  /* r: 0 or 1 = Eq. 5 on whole blocks; 2, 4 or 8 = the
                          sub-block envelope (see below) */
} eta_params_t;

/* Sub-block envelope. The pages name a "sub-block envelope" as the remedy for
 * variance dilution under flat block variance (Table 16 caption; Table 12's
 * header for the 1.45B model at b = 64) and do not define it. Reading taken
 * here: with sub_blocks = r > 1 every block of b tokens is seen as r
 * sub-blocks of b/r consecutive tokens, each with its own metadata; a block's
 * score is the largest Eq. 5 score of its sub-blocks and the admission rule is
 * unchanged. The metadata arrays then hold capacity / (b/r) columns per
 * (batch row, kv head), built by eta_build_block_meta called with a shape
 * whose block_size is b/r over sub-block ranges. Requires b/r >= 16; not
 * available for paged stores (ETA_ERR_UNSUPPORTED). The scores output holds
 * the envelope score per block. */

/* Logit gate of the decode (the current token t is exempt from both):
 * ETA_GATE_SIGMOID  g_s = S_s * sigmoid(beta (S_s - tau))   (Eq. 2-3; the pages'
 *                   "normal mode", multiplicative gating)
 * ETA_GATE_HARD     g_s = S_s if S_s >= tau, else -infinity: keys below the
 *                   threshold are removed (the "strict mode" of Tables 6-7,
 *                   hard additive masking; beta unused) */
enum { ETA_GATE_SIGMOID = 0, ETA_GATE_HARD = 1 };

/* A paged KV store: the K and V pools are [num_pages][Hkv][block_size][d]
 * (one page holds one block of every kv head) and row b's logical block j
 * lives in page block_table[b * (capacity / block_size) + j]. capacity is the
 * logical capacity of a row. A page index outside [0, num_pages) is never
 * read: the block is skipped and ETA_ERR_INVALID_ARG is recorded in the
 * device status word (by the decode; the metadata build leaves the block's
 * metadata as it was). */
typedef struct {
  const int32_t* block_table;  /* [B][capacity / block_size] int32, device memory */
  int32_t num_pages;
} eta_pages_t;

/* Block metadata of Methodology §4 ("Dual Probabilistic-Geometric Block
 * Index"): population centroid, coordinate-wise population variance and
 * maximum key norm of each full block. Layout in the conventions above. */
typedef struct {
  float* mu;
  float* var;
  float* maxnorm;
} eta_meta_t;

/* Optional screening outputs (any field may be NULL).
 *   active_idx [B][Hq][nb_cap]  ascending admitted block indices per query head
 *   active_cnt [B][Hq]          their count
 *   union_list [B][Hkv][nb_cap] ascending blocks admitted by any head of the
 *                               group, packed (block << 8) | head mask, bit g
 *                               set when query head h*G + g admitted it
 *   union_cnt  [B][Hkv]         their count
 *   scores     [B][Hq][nb_cap]  the Eq. 5 score of every screened block */
typedef struct {
  int32_t* active_idx;
  int32_t* active_cnt;
  uint32_t* union_list;
  int32_t* union_cnt;
  float* scores;
} eta_screen_out_t;

/* ABI version this library was built with (ETA_ABI_VERSION). */
ETA_API int eta_abi_version(void);

/* Short static description of a status code. */
ETA_API const char* eta_status_string(eta_status_t status);

/*
 * eta_build_block_meta — Methodology §4, block index of Eq. 5: for every
 * (batch, kv head) and every block j in [blk_begin, blk_end), write
 *   mu_i  = (sum_r k_ri) / b            (sum in increasing r, fp32)
 *   var_i = (sum_r (k_ri - mu_i)^2) / b (fused multiply-adds in increasing r)
 *   M     = sqrt(max_r sum_i k_ri^2)    (fused multiply-adds in increasing i)
 * over the block's b keys. Call it when blocks become full (after an append);
 * the partial last block never needs metadata (it is always admitted).
 *   shape  : the cache shape (q_dtype ignored)
 *   k      : K cache, kv_dtype, 16-byte aligned
 *   meta   : outputs; entries of other blocks are left untouched
 * Errors: ETA_ERR_INVALID_ARG when blk_begin < 0, blk_end > capacity/b or
 * a pointer is null/misaligned. An empty range is a no-op.
 */
ETA_API eta_status_t eta_build_block_meta(const eta_shape_t* shape, const void* k, int64_t blk_begin,
                                          int64_t blk_end, eta_meta_t meta, eta_stream_t stream);

/*
 * eta_predict_tau — Methodology §1, Eq. 1: tau[b][h] = qbar_b . W[:, h] + bias[h],
 * qbar_b the concatenation of the Hq query heads of batch b (length Hq*d).
 *   q    : [B][Hq][d] q_dtype
 *   W    : [Hq*d][Hq] fp32 row-major (W[j][h] at j*Hq + h)
 *   bias : [Hq] fp32
 *   tau  : [B][Hq] fp32 out
 * The dot product is summed in a fixed order (32 strided fp32 partials by
 * fused multiply-add, then a pairwise tree), so equal inputs give equal
 * thresholds on every run.
 */
ETA_API eta_status_t eta_predict_tau(const eta_shape_t* shape, const void* q, const float* W,
                                     const float* bias, float* tau, eta_stream_t stream);

/* Workspace bytes that eta_screen / eta_decode_sparse / eta_decode_dense need
 * for this shape (sized for the full capacity) and params (n_splits; 0 is
 * resolved on the current device). Returns 0 for an invalid shape. */
ETA_API size_t eta_decode_workspace_bytes(const eta_shape_t* shape, const eta_params_t* params);

/* Zero the workspace header (stream-ordered): the device status word and the
 * per-(batch, kv head) counters of split partials that the decode kernel
 * leaves at zero after every complete call. Call once after allocating a
 * workspace. After a call whose device status was not ETA_OK,
 * eta_read_device_status clears the header again. ws_bytes below the header
 * size (33,024 bytes) gives ETA_ERR_WORKSPACE. */
ETA_API eta_status_t eta_workspace_init(void* workspace, size_t ws_bytes, eta_stream_t stream);

/*
 * eta_screen — Methodology §4, Eq. 5 and the admission rule: for each query
 * head, score every block j < nb - n_local with
 *   Score = fl(fl(min(A, C)) * s),  A = D + z*sqrt(V),  C = sqrt(Q)*M_j,
 *   D = sum_i q_i mu_ji, V = sum_i (q_i q_i) var_ji, Q = sum_i q_i q_i
 * (fused multiply-adds in increasing i, s = 1/sqrt(d) rounded to fp32), and
 * admit the block unless Score < tau - a. The last n_local blocks are
 * admitted unscreened. Admitted lists are ascending; the union over a GQA
 * group is formed for loading (a block is read once if any head of its group
 * admits it).
 *   q        : [B][Hq][d]; tau: thresholds (see conventions), fp32
 *   meta     : written by eta_build_block_meta for every screened block
 *   out      : optional outputs (may be NULL)
 *   workspace: at least eta_decode_workspace_bytes, 256-byte aligned
 */
ETA_API eta_status_t eta_screen(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                eta_meta_t meta, int64_t n_tokens, const float* tau, int64_t tau_batch_stride,
                                const eta_screen_out_t* out, void* workspace, size_t ws_bytes,
                                eta_stream_t stream);

/*
 * eta_decode_sparse — one decode step of ETA (Figure 1 right, Figure 6):
 * screen (as eta_screen), then a flash-decoding pass over the admitted blocks
 * only, whose split partials are merged in the same kernel. For query head h
 * over the tokens s < n of its admitted blocks (Eq. 2-3):
 *   S_s = <q, k_s> / sqrt(d)
 *   g_s = S_s if s = t, else S_s * sigmoid(beta * (S_s - tau))
 *   out = sum_s exp(g_s - max g) v_s / sum_s exp(g_s - max g)       (fp32)
 * The gate uses tau; the screen uses tau - a.
 *   extra : optional screening outputs (may be NULL)
 */
ETA_API eta_status_t eta_decode_sparse(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                       const void* k, const void* v, eta_meta_t meta, int64_t n_tokens,
                                       const float* tau, int64_t tau_batch_stride, float* out,
                                       const eta_screen_out_t* extra, void* workspace, size_t ws_bytes,
                                       eta_stream_t stream);

/*
 * eta_screen_predict — eta_predict_tau and eta_screen in one launch
 * (Methodology §1 Eq. 1, then §4 Eq. 5): every screening thread block forms
 * the thresholds of its own query-head group from q, W and bias, with exactly
 * eta_predict_tau's arithmetic and order, and screens against tau - a.
 *   W, bias : as eta_predict_tau
 *   tau_out : [B][Hq] fp32 out, the thresholds (bit-identical to
 *             eta_predict_tau's); pass it to eta_decode_screened with a
 *             batch stride of Hq
 * Other arguments, outputs and errors as eta_screen.
 */
ETA_API eta_status_t eta_screen_predict(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                        eta_meta_t meta, int64_t n_tokens, const float* W, const float* bias,
                                        float* tau_out, const eta_screen_out_t* out, void* workspace,
                                        size_t ws_bytes, eta_stream_t stream);

/*
 * eta_decode_sparse_predict — one decode step with learned thresholds
 * (Eq. 1-5): eta_screen_predict, then the decode of eta_decode_sparse gated
 * by the thresholds it formed. Two launches; the result equals
 * eta_predict_tau followed by eta_decode_sparse with tau_batch_stride = Hq.
 *   tau_out : [B][Hq] fp32 out, the thresholds
 */
ETA_API eta_status_t eta_decode_sparse_predict(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                               const void* k, const void* v, eta_meta_t meta, int64_t n_tokens,
                                               const float* W, const float* bias, float* tau_out, float* out,
                                               const eta_screen_out_t* extra, void* workspace, size_t ws_bytes,
                                               eta_stream_t stream);

/*
 * eta_decode_screened — the decode half of eta_decode_sparse:
 * attend over the union lists that the last eta_screen call wrote into this
 * workspace. That call must have used the same shape, params, q, n_tokens
 * and tau (the gate reads tau here); with them, eta_screen followed by
 * eta_decode_screened gives exactly eta_decode_sparse's result. Lets a caller
 * inspect the admitted sets (counts, density) before paying for the loads.
 */
ETA_API eta_status_t eta_decode_screened(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                         const void* k, const void* v, int64_t n_tokens, const float* tau,
                                         int64_t tau_batch_stride, float* out, void* workspace, size_t ws_bytes,
                                         eta_stream_t stream);

/*
 * eta_decode_dense — the same decode kernel with every block admitted (no
 * screen, no metadata read). tau may be NULL, meaning -infinity: the gate is
 * then the identity and the result is plain softmax attention.
 */
ETA_API eta_status_t eta_decode_dense(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                      const void* k, const void* v, int64_t n_tokens, const float* tau,
                                      int64_t tau_batch_stride, float* out, void* workspace, size_t ws_bytes,
                                      eta_stream_t stream);

/*
 * Per-row lengths. The four calls below are eta_screen / eta_decode_sparse /
 * eta_decode_screened / eta_decode_dense for a batch whose rows hold
 * different numbers of cached tokens (the paged or continuous-batching case):
 *   seq_lens   : [B] int32, device memory: tokens of row b including its
 *                current token (t_b = seq_lens[b] - 1). Rows attend, screen
 *                and are gated exactly as a call with n_tokens = seq_lens[b].
 *                Read on the device, so a CUDA graph can replay the call
 *                while the lengths change.
 *   max_tokens : host upper bound of seq_lens, 1 <= max_tokens <= capacity;
 *                sizes the launches. A length outside [1, max_tokens] sets
 *                ETA_ERR_INVALID_ARG in the device status word and is clamped
 *                to that range.
 * Thresholds (eta_screen_ragged, eta_decode_sparse_ragged): with W == NULL
 * they are tau / tau_batch_stride as in eta_screen; with W set they are
 * formed by Eq. 1 as in eta_screen_predict (tau ignored, tau_out [B][Hq]
 * written). Other arguments, outputs and errors as the uniform-length calls.
 */
ETA_API eta_status_t eta_screen_ragged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                       eta_meta_t meta, const int32_t* seq_lens, int64_t max_tokens,
                                       const float* tau, int64_t tau_batch_stride, const float* W,
                                       const float* bias, float* tau_out, const eta_screen_out_t* out,
                                       void* workspace, size_t ws_bytes, eta_stream_t stream);
ETA_API eta_status_t eta_decode_sparse_ragged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                              const void* k, const void* v, eta_meta_t meta,
                                              const int32_t* seq_lens, int64_t max_tokens, const float* tau,
                                              int64_t tau_batch_stride, const float* W, const float* bias,
                                              float* tau_out, float* out, const eta_screen_out_t* extra,
                                              void* workspace, size_t ws_bytes, eta_stream_t stream);
ETA_API eta_status_t eta_decode_screened_ragged(const eta_shape_t* shape, const eta_params_t* params,
                                                const void* q, const void* k, const void* v,
                                                const int32_t* seq_lens, int64_t max_tokens, const float* tau,
                                                int64_t tau_batch_stride, float* out, void* workspace,
                                                size_t ws_bytes, eta_stream_t stream);
ETA_API eta_status_t eta_decode_dense_ragged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                             const void* k, const void* v, const int32_t* seq_lens,
                                             int64_t max_tokens, const float* tau, int64_t tau_batch_stride,
                                             float* out, void* workspace, size_t ws_bytes, eta_stream_t stream);

/*
 * Paged KV (see eta_pages_t): the per-row-length calls on K and V pools
 * addressed through a block table, with per-row lengths (seq_lens,
 * max_tokens) as in eta_decode_sparse_ragged. The metadata stays indexed by
 * logical block ([B][Hkv][d][capacity / block_size]); eta_build_block_meta_paged
 * builds it from the pool. A row's result equals the contiguous call on the
 * cache its pages describe, bit for bit.
 */
ETA_API eta_status_t eta_build_block_meta_paged(const eta_shape_t* shape, const void* k_pool, eta_pages_t pages,
                                                int64_t blk_begin, int64_t blk_end, eta_meta_t meta,
                                                eta_stream_t stream);
ETA_API eta_status_t eta_decode_sparse_paged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                             const void* k_pool, const void* v_pool, eta_pages_t pages,
                                             eta_meta_t meta, const int32_t* seq_lens, int64_t max_tokens,
                                             const float* tau, int64_t tau_batch_stride, const float* W,
                                             const float* bias, float* tau_out, float* out,
                                             const eta_screen_out_t* extra, void* workspace, size_t ws_bytes,
                                             eta_stream_t stream);
ETA_API eta_status_t eta_decode_screened_paged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                               const void* k_pool, const void* v_pool, eta_pages_t pages,
                                               const int32_t* seq_lens, int64_t max_tokens, const float* tau,
                                               int64_t tau_batch_stride, float* out, void* workspace,
                                               size_t ws_bytes, eta_stream_t stream);
ETA_API eta_status_t eta_decode_dense_paged(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                            const void* k_pool, const void* v_pool, eta_pages_t pages,
                                            const int32_t* seq_lens, int64_t max_tokens, const float* tau,
                                            int64_t tau_batch_stride, float* out, void* workspace, size_t ws_bytes,
                                            eta_stream_t stream);

/*
 * eta_block_stats — the measurements behind the screen diagnostics of
 * Table 16 (false negatives, false positives, token recall, missed mass). A
 * dense pass over K (not a decode step): for every query head h and block
 * j < ceil(n_tokens / block_size), with S_s = fl(fl(sum_i q_i k_si) * s) (fused
 * multiply-adds in increasing i, s = fl(1/sqrt(d))):
 *   block_max[b][h][j] = max over the block's tokens of S_s
 *   above[b][h][j]     = tokens of the block with S_s >= tau - a
 *   block_lse[b][h][j] = log sum over the block's tokens of exp(g_s), g_s the
 *                        gated logit of params->gate with threshold tau (the
 *                        current token exempt)
 * Outputs are [B][Hq][capacity / block_size] fp32 / int32 / fp32; entries of
 * blocks past n_tokens are left untouched. The maxima and counts are
 * reproducible bit for bit; a block is "truly active" when its max reaches
 * tau - a, and the fraction of gated softmax mass in the blocks a screen
 * rejected is sum_rejected exp(lse_j) / sum_all exp(lse_j).
 */
ETA_API eta_status_t eta_block_stats(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                     const void* k, int64_t n_tokens, const float* tau, int64_t tau_batch_stride,
                                     float* block_max, int32_t* above, float* block_lse, eta_stream_t stream);

/*
 * eta_screen_diagnostics — Table 16's screen quality per query head, from the
 * outputs of eta_block_stats (block_max, above, block_lse) and of eta_screen
 * (active_idx, active_cnt) for the same shape, params, n_tokens and tau. Over
 * a head's screened blocks j < ceil(n_tokens / b) - n_local, a block is "truly
 * active" when block_max[j] >= fl(tau - a):
 *   per_head[b][h][0] false negatives: truly active blocks not admitted / truly active
 *   per_head[b][h][1] false positives: admitted blocks not truly active / admitted
 *   per_head[b][h][2] token recall:    sum of above over admitted blocks / over all
 *   per_head[b][h][3] missed mass:     sum of exp(block_lse) over rejected blocks /
 *                                      over every block (fp64)
 * A zero denominator counts as one. per_head: [B][Hq][4] fp64, 8-byte aligned.
 */
ETA_API eta_status_t eta_screen_diagnostics(const eta_shape_t* shape, const eta_params_t* params, int64_t n_tokens,
                                            const float* tau, int64_t tau_batch_stride, const float* block_max,
                                            const int32_t* above, const float* block_lse, const int32_t* active_idx,
                                            const int32_t* active_cnt, double* per_head, eta_stream_t stream);

/*
 * eta_decode_sparse_static — eta_decode_sparse without a caller workspace and
 * without any device allocation. The paper has no counterpart: this entry
 * point exists for callers that cannot allocate device memory when they
 * decode: a serving engine whose memory plan is frozen at start-up, a host
 * framework that owns every allocation and hands out only finished tensors,
 * a real-time loop that must not enter an allocator (cudaMalloc may
 * synchronise the device and has no latency bound).
 *
 * The scratch is a fixed array of ETA_STATIC_SCRATCH_BYTES inside the library,
 * one per device that loads it, held until the process exits. Shapes whose
 * eta_decode_workspace_bytes exceeds that size are rejected with
 * ETA_ERR_WORKSPACE before anything is launched. All calls on a device share
 * the array: calls whose kernels overlap on the GPU (unordered streams) race
 * and must not be issued. The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress); make it before any stream capture.
 * Each call clears the scratch header (status word and partial counters)
 * first. device_status (nullable,
 * device memory) receives this call's device status word, stream-ordered.
 * Other arguments and results as eta_decode_sparse.
 */
#define ETA_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
ETA_API eta_status_t eta_decode_sparse_static(const eta_shape_t* shape, const eta_params_t* params, const void* q,
                                              const void* k, const void* v, eta_meta_t meta, int64_t n_tokens,
                                              const float* tau, int64_t tau_batch_stride, float* out,
                                              const eta_screen_out_t* extra, int32_t* device_status,
                                              eta_stream_t stream);

/*
 * eta_test_withhold_copy — test hook of the device-timeout path; the paper has
 * no counterpart. The next decode launch in this process (any eta_decode_*
 * call) leaves the K/V copy of one admitted block unissued: position
 * `position` (0-based) of the first thread block's range. The consumer warp
 * that owns that block waits for it up to the library's device wait limit
 * (2 s), then every warp of that thread block stops, the copies already
 * issued are allowed to land, and the call records ETA_ERR_DEVICE_TIMEOUT in
 * the workspace status word; its outputs are then undefined. Nothing faults
 * and the context stays usable: read (and so clear) the status with
 * eta_read_device_status, and the next call computes normally. A position
 * past the end of that range withholds nothing; a negative position disarms
 * the hook. Always returns ETA_OK. Not for production use.
 */
ETA_API eta_status_t eta_test_withhold_copy(int64_t position);

/* Synchronise `stream`, read the workspace's device status word into *status
 * (host pointer) and clear it (the whole header when it was not ETA_OK).
 * Returns ETA_ERR_CUDA if the copy fails. */
ETA_API eta_status_t eta_read_device_status(const void* workspace, eta_stream_t stream, eta_status_t* status);

#ifdef __cplusplus
}
#endif

#endif /* ETA_H_ */
