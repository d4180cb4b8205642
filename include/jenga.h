/*
 * jenga.h -- C ABI of the token-sparse layer library (B200, sm_100a).
 *
 * The operations follow the Jenga paper ("Jenga: Enhancing LLM Long-Context
 * Fine-tuning with Contextual Token Sparsity", ATC'25), as described by the
 * papercache.org deep notes ("Jenga notes") and the aipaper.cc summary ("Jenga
 * summary"):
 *   - block informativeness scoring      Jenga summary §4.2.1 Eq. (1), §4.2.2 Eq. (2), §4.2.3
 *   - threshold selection                Jenga notes §4.2 Algorithm 1; Jenga summary §4.2.3
 *   - permutation-free gather / in-place residual scatter-add
 *                                        Jenga notes §4.4; Jenga summary §4.4.1 (Fig. 9)
 *   - retained-token layer forward/backward, segment-wise gradients
 *                                        Jenga summary §4.1 (Fig. 5), §4.4.2 (Fig. 10)
 *   - block-score predictor              Jenga notes §4.3; Jenga summary §4.3.1 (Fig. 8)
 *
 * Conventions
 * -----------
 *  * Every function returns jenga_status; none aborts.  jenga_last_error() gives
 *    the text of the last failure on the calling host thread.
 *  * All tensor pointers are CALLER-OWNED DEVICE memory.  The library never
 *    allocates or frees device memory; scratch space is passed in as a workspace
 *    whose size is given by the matching *_workspace_bytes / *_bytes query.
 *  * Every call is asynchronous on the given CUDA stream (NULL = legacy default
 *    stream) and does not synchronise the host.  Argument checks that need only
 *    host values are done before launch (JENGA_EINVAL).  Faults that only the
 *    device can see (an index out of range, an n_kept above the stated maximum, a
 *    pipeline wait that ran past its time budget) are recorded in a device error
 *    word; jenga_check_device_status() synchronises the stream, reads and clears it.
 *  * Layouts are row-major.  Activations are token-major [B, S, hidden]; per-head
 *    tensors are [B, S, H, D] (a token's H*D values contiguous, token pitch ld);
 *    weights are [out, in] (PyTorch Linear).  bf16 = IEEE bfloat16 bits.
 *  * Block indices are int32, ascending, kept blocks first; entries past n_kept
 *    are -1.  Token t of kept block i (0 <= t < blk) is sequence row
 *    idx[i] * blk + t and compact row i * blk + t.
 */
#ifndef JENGA_H_
#define JENGA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define JENGA_API __attribute__((visibility("default")))
#else
#define JENGA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* jenga_stream_t; /* same object as cudaStream_t */

typedef enum {
  JENGA_OK = 0,
  JENGA_EINVAL = 1,       /* bad argument (shape, pointer, mode) */
  JENGA_EUNSUPPORTED = 2, /* valid but not implemented for these sizes / dtypes */
  JENGA_ECUDA = 3,        /* a CUDA runtime call failed */
  JENGA_ETIMEOUT = 4,     /* a device-side wait ran past its budget */
  JENGA_EWORKSPACE = 5,   /* workspace / saved buffer smaller than required */
  JENGA_EINTERNAL = 6,    /* device detected an internal inconsistency (bad index) */
} jenga_status;

typedef enum { JENGA_F32 = 0, JENGA_BF16 = 1 } jenga_dtype;

typedef enum {
  /* Jenga summary §4.2.1 Eq. (1) with S_ij the causal softmax probability of query i on
   * key j (diagonal included), summed over queries and heads (no 1/N_head), then over
   * the tokens of each key block (§4.2.3).  Per sequence the scores sum to H * S. */
  JENGA_SCORE_SOFTMAX_MASS = 0,
  /* Jenga summary §4.2.2 Eq. (2): for each (query block, key block) score block the
   * max over causal entries of sum_h max(q_i.k_j/sqrt(D), 0) / N_head, summed over
   * query blocks (§4.2.3). */
  JENGA_SCORE_PAPER_BLOCKMAX = 1,
} jenga_score_mode;

typedef enum {
  JENGA_SELECT_MEAN_GE = 0,   /* keep score >= average block score (Algorithm 1, step 1) */
  JENGA_SELECT_TOPK_FRAC = 1, /* keep k = ceil(param * nb - 1e-6) blocks, rank (score desc, index asc) */
  JENGA_SELECT_ABS_GE = 2,    /* keep score >= param */
  JENGA_SELECT_TOPK = 3,      /* keep k = (int)param blocks, same ranking */
} jenga_select_mode;

/* ------------------------------------------------------------------ status */
JENGA_API const char* jenga_status_string(jenga_status st);
/* Copies the last error message of this host thread (NUL-terminated, truncated). */
JENGA_API size_t jenga_last_error(char* buf, size_t len);
/* Synchronises `stream`, returns the first device-recorded fault since the last call
 * (JENGA_OK if none) and clears it.  detail (nullable) gets {site, info}. */
JENGA_API jenga_status jenga_check_device_status(jenga_stream_t stream, uint32_t* detail2);
/* Device-side wait budget in nanoseconds for every pipeline wait (default 2e9).
 * Applies to launches made after the call. */
JENGA_API jenga_status jenga_set_wait_budget_ns(uint64_t ns);
/* Library version and build string. */
JENGA_API const char* jenga_version(void);
/* Launch timing for measurement: while enabled, every kernel the library launches is
 * bracketed by two CUDA events recorded on the launch's own stream (host-thread
 * local use; no device memory).  Enabling clears previous records. */
JENGA_API jenga_status jenga_profile_enable(int on);
/* Waits for the recorded events, writes {"kernel": {"launches": n, "ms": total}, ...}
 * (NUL-terminated, truncated to len) and clears the records; returns the full length. */
JENGA_API size_t jenga_profile_report(char* buf, size_t len);

/* ------------------------------------------------------------------ scoring
 * jenga_score_blocks -- block informativeness (a2 + a3 of the path).
 *   q, k     : [B, S, H, D] of dtype dt; token pitch ldq / ldk elements (>= H*D),
 *              batch pitch S * ld.  q and k may alias one fused [S, 2*H*D] buffer.
 *   blk      : tokens per block, S % blk == 0; nb = S / blk.
 *   causal   : 1 = query i attends keys j <= i (the scoring the path uses); 0 = all j.
 *   scores   : [B, nb] fp32 out.  Deterministic (fixed reduction order).
 *   ws       : workspace of jenga_score_workspace_bytes(...) bytes.  After a softmax-mass
 *              call its first B*H*S floats (from the first 256-byte aligned address of ws)
 *              hold the negated row log-sum-exp -log2 sum_{j<=i} 2^(log2(e) q_i.k_j/sqrt(D))
 *              of every (sequence, head, query), a diagnostic; the rest is scratch.
 * fp32 inputs use exact fp32 SIMT dot products (D <= 128).  bf16 inputs use the single-pass
 * tensor-core kernel and need D == 128 and blk a multiple of 32 (S itself need not be a
 * multiple of the 128-token tile).  Errors: EINVAL (shapes), EWORKSPACE, EUNSUPPORTED
 * (D / dtype / blk / mode combination not built). */
JENGA_API size_t jenga_score_workspace_bytes(int B, int S, int H, int D, int blk);
JENGA_API jenga_status jenga_score_blocks(const void* q, int64_t ldq, const void* k, int64_t ldk, int B, int S, int H,
                                int D, int blk, int causal, jenga_dtype dt, jenga_score_mode mode,
                                float* scores, void* ws, size_t ws_bytes, jenga_stream_t stream);

/* jenga_score_blocks_noalloc -- jenga_score_blocks without a workspace argument.
 * (The paper has no counterpart: this is an interface convenience.)  For callers that
 * cannot hand the library device scratch memory -- hosts that own all device memory and
 * allow no allocation outside their own pool, or latency-critical code that cannot
 * afford cudaMalloc / cudaFree and the device synchronisation they may cause.  The
 * scratch is one fixed 16 MiB array inside the library image (every GPU that loads the
 * library holds it until the process exits).  Limit: jenga_score_workspace_bytes(B, S, H,
 * D, blk) must not exceed jenga_score_blocks_noalloc_max_bytes(); larger sizes return
 * JENGA_EWORKSPACE before anything is launched.  That covers every mode: the fp32 path
 * needs 2*B*H*S*4 bytes, the bf16 single pass about 4*B*H*S*(1 + S/(64*128)) bytes plus
 * 512*(S/64 + 8) bytes per work slot (at most 160 slots), the block-max mode
 * 4*B*(S/g)^2 bytes (g = blk for blk 32 or 64, else 128); e.g. 32 heads of 128 with blocks
 * of 64 fit up to S = 8192.
 * Arguments and results are those of jenga_score_blocks.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress, that device current), and so
 * does the first call in a new CUDA context of that device (after a device reset): make
 * such a first call before any stream capture.  All calls share the array and each call
 * overwrites what it reads, so nothing needs clearing, but calls whose kernels overlap on
 * the GPU (for example on two streams) race on it.  Allocates nothing.
 * jenga_score_blocks_noalloc_max_bytes() returns the array size in bytes. */
JENGA_API size_t jenga_score_blocks_noalloc_max_bytes(void);
JENGA_API jenga_status jenga_score_blocks_noalloc(const void* q, int64_t ldq, const void* k, int64_t ldk, int B,
                                                  int S, int H, int D, int blk, int causal, jenga_dtype dt,
                                                  jenga_score_mode mode, float* scores, jenga_stream_t stream);

/* ------------------------------------------------------------------ selection
 * jenga_select -- threshold / top-k selection and compaction (a4).
 *   scores : [B, nb] fp32 (NaN compares as -inf).
 *   idx    : [B, nb] int32 out, ascending kept block indices then -1.
 *   n_kept : [B] int32 out.   mask : [B, nb] uint8 out (nullable).
 *   ws     : jenga_select_workspace_bytes(B, nb) bytes (0 for nb <= 8192).
 * MEAN_GE forms the average as a float64 sum of the scores divided by nb and
 * compares each score as float64.  TOPK modes are exact (rank counting).  Large nb
 * (> 8192) supports MEAN_GE and ABS_GE (multi-CTA ballot + prefix-sum compaction). */
JENGA_API size_t jenga_select_workspace_bytes(int B, int nb);
JENGA_API jenga_status jenga_select(const float* scores, int B, int nb, jenga_select_mode mode, float param,
                          int32_t* idx, int32_t* n_kept, uint8_t* mask, void* ws, size_t ws_bytes,
                          jenga_stream_t stream);

/* ------------------------------------------------------------------ token movement
 * jenga_gather -- out[b, i*blk + t, :] = x[b, idx[b,i]*blk + t, :] for i < n_kept[b] (a5).
 *   x   : [B, S, h] (row pitch ldx elements), out : [B, n_cap, h] (row pitch ldo),
 *   n_cap = rows of out per batch (>= n_kept[b]*blk, checked on device).  Rows of out
 *   past n_kept[b]*blk are not written.  dt: F32 or BF16.  h * elem % 16 == 0 and
 *   16-byte aligned rows use 128-bit moves. */
JENGA_API jenga_status jenga_gather(const void* x, int64_t ldx, int B, int S, int h, int blk, const int32_t* idx,
                          const int32_t* n_kept, jenga_dtype dt, void* out, int64_t ldo, int n_cap,
                          jenga_stream_t stream);

/* jenga_scatter_add -- in-place residual add of a retained-row result (a7):
 *   x[b, idx[b,i]*blk + t, :] = round(x + alpha * y[b, i*blk + t, :]); other rows untouched.
 *   The sum is one fp32 fused multiply-add, rounded once more to bf16 for bf16 data. */
JENGA_API jenga_status jenga_scatter_add(void* x, int64_t ldx, const void* y, int64_t ldy, int B, int S, int h, int blk,
                               const int32_t* idx, const int32_t* n_kept, float alpha, jenga_dtype dt,
                               int n_cap, jenga_stream_t stream);

/* jenga_scale_rows -- x[b, rows[b,i], :] *= factor for i < n_rows (salient-token
 * emphasis of synthetic inputs, and its backward as the same diagonal). */
JENGA_API jenga_status jenga_scale_rows(void* x, int64_t ldx, int B, int S, int h, const int32_t* rows, int n_rows,
                              float factor, jenga_dtype dt, jenga_stream_t stream);

/* ------------------------------------------------------------------ layer
 * A Llama-2 decoder layer (RMSNorm -> q/k/v with RoPE -> causal attention -> o_proj
 * -> residual; RMSNorm -> SiLU-gated MLP -> residual) with LoRA on q_proj and v_proj,
 * run only on the retained rows (Jenga summary §4.1, §4.4.1).  bf16 storage, fp32
 * accumulation.  RoPE uses each token's ORIGINAL position (rotate-half, pairs d and
 * d + D/2, angle pos * theta^(-2i/D)); attention is causal among retained tokens.
 * head_dim must be 128, heads at most 64 with heads * 128 a multiple of 256, hidden a
 * multiple of 256 up to 8192, ffn a multiple of 256, lora rank 16. */
typedef struct jenga_layer_weights {
  int hidden, heads, head_dim, ffn;
  float rms_eps, rope_theta;
  const void* attn_norm; /* [hidden] bf16 RMSNorm gain before attention */
  const void* mlp_norm;  /* [hidden] bf16 RMSNorm gain before the MLP */
  const void* wq;        /* [H*D, hidden] bf16 */
  const void* wk;        /* [H*D, hidden] bf16 */
  const void* wv;        /* [H*D, hidden] bf16 */
  const void* wo;        /* [hidden, H*D] bf16 */
  const void* wg;        /* [ffn, hidden] bf16 gate_proj */
  const void* wu;        /* [ffn, hidden] bf16 up_proj */
  const void* wd;        /* [hidden, ffn] bf16 down_proj */
} jenga_layer_weights;

typedef struct jenga_lora {
  int rank;       /* 16 */
  float scale;    /* alpha / rank */
  const void* aq; /* [rank, hidden] bf16 */
  const void* bq; /* [H*D, rank] bf16 */
  const void* av; /* [rank, hidden] bf16 */
  const void* bv; /* [H*D, rank] bf16 */
} jenga_lora;

typedef struct jenga_lora_grads { /* fp32, ACCUMULATED into (+=) */
  float* daq;                     /* [rank, hidden] */
  float* dbq;                     /* [H*D, rank] */
  float* dav;
  float* dbv;
} jenga_lora_grads;

/* Packed (re-laid-out) copies of the frozen weights the kernels read: fused QKV,
 * gate/up interleaved in 64-row groups, and the transposes the backward needs.  The
 * backward's copies (the transposes of Wo, Wq | Wk | Wv and [Wg; Wu], and of the LoRA
 * matrices) are fp16, because the backward products run on fp16 operands: a weight whose
 * magnitude exceeds 65504 (fp16's largest finite value) makes jenga_check_device_status
 * report JENGA_EINVAL (site 9, detail = element index).  The LoRA matrices are read at pack
 * time: pack again after changing them.  The LoRA operand of the dX product is divided by
 * a power of two chosen here from Bq, Bv and lora->scale, which keeps it in fp16's range
 * for a backward LoRA scale up to max(lora->scale, 1).
 * Built once per layer with jenga_layer_pack; read-only afterwards. */
JENGA_API size_t jenga_layer_pack_bytes(const jenga_layer_weights* w, const jenga_lora* lora);
JENGA_API jenga_status jenga_layer_pack(const jenga_layer_weights* w, const jenga_lora* lora, void* packed,
                              size_t packed_bytes, jenga_stream_t stream);

/* jenga_layer_score_qk -- a1: q and k of ALL S tokens for scoring (no grad):
 *   qk[b, s, 0:H*D] = RoPE(RMSNorm(x) Wq^T + scale (RMSNorm(x) Aq^T) Bq^T)
 *   qk[b, s, H*D:2*H*D] = RoPE(RMSNorm(x) Wk^T), positions s.  qk: [B, S, 2*H*D] bf16. */
JENGA_API size_t jenga_layer_score_qk_workspace_bytes(const jenga_layer_weights* w, int B, int S);
JENGA_API jenga_status jenga_layer_score_qk(const jenga_layer_weights* w, const jenga_lora* lora, const void* packed,
                                  const void* x, int B, int S, void* qk, void* ws, size_t ws_bytes,
                                  jenga_stream_t stream);

/* jenga_sparse_layer_fwd -- a5 + a6 + a7: the layer on the kept blocks of x, in place.
 *   x      : [B, S, hidden] bf16, updated in place on retained rows only.
 *   idx, n_kept : from jenga_select; n_kept_max: host bound on every n_kept[b].
 *   saved  : jenga_layer_saved_bytes(...) bytes; written here, read by the backward.  It
 *            holds, per retained row, the gathered input, q | k | v, the attention output,
 *            the residual h, the MLP pre-activations (gate, up) in fp16 (so the backward
 *            does not recompute them; a pre-activation above 65504 in magnitude becomes
 *            infinite there), the LoRA down-projections and the row statistics.
 *   ws     : jenga_layer_fwd_workspace_bytes(...) bytes of scratch. */
JENGA_API size_t jenga_layer_saved_bytes(const jenga_layer_weights* w, int B, int blk, int n_kept_max);
JENGA_API size_t jenga_layer_fwd_workspace_bytes(const jenga_layer_weights* w, int B, int blk, int n_kept_max);
JENGA_API jenga_status jenga_sparse_layer_fwd(const jenga_layer_weights* w, const jenga_lora* lora, const void* packed,
                                    void* x, int B, int S, int blk, const int32_t* idx, const int32_t* n_kept,
                                    int n_kept_max, void* saved, size_t saved_bytes, void* ws, size_t ws_bytes,
                                    jenga_stream_t stream);

/* jenga_sparse_layer_fwd_qk -- jenga_sparse_layer_fwd that takes the retained rows' q and k
 * from qk_all, the [S, 2 H D] bf16 post-RoPE q | k of all rows that jenga_layer_score_qk
 * produced for scoring from the same x (row pitch ld_qk elements, 16-byte aligned rows;
 * read only), and projects only v (+ LoRA-v): the same kernels made those q and k, so the
 * result is bit-identical to jenga_sparse_layer_fwd.  qk_all must be recomputed after ANY
 * change to x (including jenga_scale_rows), to the weights or to the LoRA tensors: the
 * library cannot detect a stale buffer, and one silently gives wrong q and k.  qk_all must
 * hold at least S rows (the library cannot check its row count).  Other arguments and
 * errors as there. */
JENGA_API jenga_status jenga_sparse_layer_fwd_qk(const jenga_layer_weights* w, const jenga_lora* lora, const void* packed,
                                       void* x, int B, int S, int blk, const int32_t* idx, const int32_t* n_kept,
                                       int n_kept_max, const void* qk_all, int64_t ld_qk, void* saved,
                                       size_t saved_bytes, void* ws, size_t ws_bytes, jenga_stream_t stream);

/* jenga_sparse_layer_fwd_mlp -- jenga_sparse_layer_fwd (or _fwd_qk when qk_all is not null)
 * with MLP-block token elimination (Jenga summary §4.2.4, extend to the MLP block): after the
 * gate / up projection of all retained rows, each retained block's MLP informativeness is the
 * L1 mass of its activation SiLU(gate) * up (jenga_mlp_block_scores), jenga_select(mlp_mode,
 * mlp_param) picks the blocks the MLP sub-block keeps among the n_kept_max retained positions
 * (TOPK_FRAC: a fraction of n_kept_max; TOPK: a count; ABS_GE: a threshold), and the down
 * projection and its in-place residual add run only on those blocks; on the other retained
 * blocks the layer output is h, the attention sub-block's output.  The keep mask is stored in
 * `saved`, and jenga_sparse_layer_bwd then runs the MLP backward (the dA GEMM with the SwiGLU
 * derivative, the dhn GEMM) only on the kept blocks and passes the upstream gradient straight
 * through the MLP branch of the others.
 *   mlp_scores : [n_kept_max] fp32 out (nullable): the criterion per retained position
 *             (-inf at and past the device count n_kept);
 *   mlp_pos : [n_kept_max] int32 out (nullable): kept positions in the retained list,
 *             ascending, then -1 (compose with idx by jenga_compose_block_indices for
 *             sequence block numbers);  n_mlp : [1] int32 out (nullable): their count.
 * n_kept_max <= 8192.  Other arguments, workspace and errors as jenga_sparse_layer_fwd. */
JENGA_API jenga_status jenga_sparse_layer_fwd_mlp(const jenga_layer_weights* w, const jenga_lora* lora,
                                                  const void* packed, void* x, int B, int S, int blk,
                                                  const int32_t* idx, const int32_t* n_kept, int n_kept_max,
                                                  const void* qk_all, int64_t ld_qk, jenga_select_mode mlp_mode,
                                                  float mlp_param, float* mlp_scores, int32_t* mlp_pos,
                                                  int32_t* n_mlp, void* saved, size_t saved_bytes, void* ws,
                                                  size_t ws_bytes, jenga_stream_t stream);

/* jenga_sparse_layer_bwd -- a8 + a9: backward of jenga_sparse_layer_fwd for an upstream
 * gradient G held in dx ([B, S, hidden] bf16).  On return dx holds dL/dx: eliminated
 * rows keep G (identity through the residual), retained rows get the layer backward.
 * Frozen base weights get no gradient; LoRA gradients are ACCUMULATED into grads.
 * The retained rows are processed in consecutive segments of segment_tokens rows
 * (multiple of 128; last one short), last segment first, so per-segment scratch is
 * bounded by the segment length (Jenga summary §4.4.2).  Precision: fp32 accumulation
 * throughout; the products with the frozen weights take the gradient rows as fp16, each
 * row scaled by the power of two that puts its largest magnitude in [2^13, 2^14) (undone
 * exactly in the product's epilogue); the attention backward runs on fp16 copies of q, k,
 * v and of the segment's dO scaled by a power of two.  Deterministic: a fixed reduction
 * order everywhere, so repeated calls give identical bits. */
JENGA_API size_t jenga_layer_bwd_workspace_bytes(const jenga_layer_weights* w, int B, int blk, int n_kept_max,
                                       int segment_tokens);
JENGA_API jenga_status jenga_sparse_layer_bwd(const jenga_layer_weights* w, const jenga_lora* lora, const void* packed,
                                    void* dx, int B, int S, int blk, const int32_t* idx, const int32_t* n_kept,
                                    int n_kept_max, const void* saved, size_t saved_bytes, jenga_lora_grads* grads,
                                    int segment_tokens, void* ws, size_t ws_bytes, jenga_stream_t stream);

/* ------------------------------------------------------------------ predictor
 * jenga_predict_blocks -- a10 (Jenga notes §4.3; Jenga summary §4.3.1): per block the
 * mean of its rows of x (raw layer input), then s = W2 . GELU(W1 xbar + b1) + b2
 * with exact-erf GELU.  x [B, S, h] bf16; W1 [m, h] bf16, b1 [m] fp32, W2 [m] bf16,
 * b2 [1] fp32 (device); scores [B, nb] fp32.  m <= 256.
 * ws: jenga_predict_workspace_bytes bytes (pooled block means, fp32). */
JENGA_API size_t jenga_predict_workspace_bytes(int B, int S, int h, int blk);
JENGA_API jenga_status jenga_predict_blocks(const void* x, int B, int S, int h, int blk, const void* w1, const float* b1,
                                  const void* w2, const float* b2, int m, float* scores, void* ws,
                                  size_t ws_bytes, jenga_stream_t stream);

/**
 * jenga_mlp_block_scores -- MLP-block elimination criterion (Jenga summary §4.2.4): the
 * informativeness of a retained token block for the MLP sub-block from the block's
 * intermediate activation a = SiLU(gate) * up:
 *   scores[i] = sum over the blk rows of block i and the F neurons of |a|,   i < *n_kept,
 *   scores[i] = -inf for n_kept <= i < n_cap (never selected).
 * a: device bf16 [n_cap * blk, F] with row pitch lda (rows in compact retained order, as
 * the layer forward forms them), 16-byte aligned, F and lda multiples of 8; n_kept:
 * device int32 (retained blocks; null = n_cap); scores: device fp32 [n_cap].  Selecting
 * on these scores (jenga_select) gives positions in the retained list; compose them with
 * jenga_compose_block_indices for sequence block numbers.  Errors: JENGA_EINVAL. */
JENGA_API jenga_status jenga_mlp_block_scores(const void* a, int64_t lda, int F, int blk, const int32_t* n_kept,
                                              int n_cap, float* scores, jenga_stream_t stream);
/* jenga_compose_block_indices -- out[i] = outer[pos[i]] for i < *n_pos, -1 for
 * *n_pos <= i < n_cap: a list of positions in the outer index list (e.g. the MLP's kept
 * positions among the attention-retained blocks) in the outer list's numbering.  All
 * device int32; an out-of-range position records JENGA_EINTERNAL and writes -1. */
JENGA_API jenga_status jenga_compose_block_indices(const int32_t* outer, int n_outer_cap, const int32_t* pos,
                                                   const int32_t* n_pos, int n_cap, int32_t* out,
                                                   jenga_stream_t stream);

/**
 * jenga_predict_blocks_qk -- the pages' Q/K predictor pair (Jenga summary §4.3.1 Eq. (3),
 * Fig. 8): a query-side and a key-side predictor, each three bias-free low-rank matrices
 * with ReLU between them, map the mean of each block's raw layer-input rows to d-vectors
 *   qhat_m = W3q ReLU(W2q ReLU(W1q xbar_m)),   khat_n = W3k ReLU(W2k ReLU(W1k xbar_n));
 * the score block (m, n) is qhat_m . khat_n and scores[b, n] is the sum of column n over
 * the query blocks m (m >= n when causal != 0).
 * x: device bf16 [B, S, h] (row pitch h, 16-byte aligned); q_w1, k_w1: bf16 [r1, h]
 * (16-byte aligned); q_w2, k_w2: bf16 [r2, r1]; q_w3, k_w3: bf16 [d, r2]; scores: device
 * fp32 [B, S / blk].  h % 8 == 0, h <= 12288, r1 and r2 in [1, 1024], d in [1, 64].
 * ws: jenga_predict_qk_workspace_bytes(B, S, h, blk, d) bytes (block means and the two
 * sides' outputs, fp32).  Errors: JENGA_EINVAL, JENGA_EWORKSPACE. */
JENGA_API size_t jenga_predict_qk_workspace_bytes(int B, int S, int h, int blk, int d);
JENGA_API jenga_status jenga_predict_blocks_qk(const void* x, int B, int S, int h, int blk, const void* q_w1,
                                               const void* q_w2, const void* q_w3, const void* k_w1,
                                               const void* k_w2, const void* k_w3, int r1, int r2, int d, int causal,
                                               float* scores, void* ws, size_t ws_bytes, jenga_stream_t stream);

/**
 * jenga_lm_loss_segmented -- causal-LM cross-entropy over the vocabulary with its
 * hidden-state gradient, computed segment by segment (Jenga summary §4.4.2, segment-based
 * peak cutting, Fig. 10): the tokens are processed segment_tokens rows at a time, so the
 * vocabulary-wide logits of only one segment exist at a time.
 *   logits_t  = hidden_t . W^T                          (W [V, h]: frozen output embedding)
 *   *loss     = (1/n) sum over valid t of (logsumexp(logits_t) - logits_t[labels[t]])
 *   dhidden_t = (1/n) (softmax(logits_t) - onehot(labels[t])) . W for valid t, else 0
 * where t is valid when 0 <= labels[t] < V (any other label, e.g. -100, is ignored) and n
 * is the number of valid tokens (loss 0 and zero gradient when n == 0).
 * hidden: device bf16 [S, h] (row pitch h); w: device bf16 [V, h]; labels: device int32
 * [S] (already shifted to the next token); loss: device fp32 scalar; dhidden: device bf16
 * [S, h] (written).  h and V multiples of 64; hidden, w, dhidden 16-byte aligned.  The
 * result does not depend on segment_tokens (each row depends only on itself).
 * ws: jenga_lm_loss_workspace_bytes(S, h, V, segment_tokens) bytes of device memory
 * (transposed W, one segment's fp32 logits and bf16 gradient rows, per-row losses); all
 * buffers are caller-owned.  Errors: JENGA_EINVAL (sizes, alignment, null), JENGA_EWORKSPACE. */
JENGA_API size_t jenga_lm_loss_workspace_bytes(int S, int h, int V, int segment_tokens);
JENGA_API jenga_status jenga_lm_loss_segmented(const void* hidden, const void* w, const int32_t* labels, int S, int h,
                                               int V, int segment_tokens, float* loss, void* dhidden, void* ws,
                                               size_t ws_bytes, jenga_stream_t stream);

/* ------------------------------------------------------------------ test hook
 * jenga_test_gemm -- C[M, N] = A[M, K] * B[N, K]^T through the tcgen05 GEMM the layer
 * uses (bf16 inputs, fp32 accumulate; C fp32 if out_f32 else bf16).  bn: 256 or 32
 * (output tile width).  K % 64 == 0; rows 16-byte aligned.  For kernel tests only. */
JENGA_API jenga_status jenga_test_gemm(const void* A, int64_t lda, const void* B, int64_t ldb, int M, int N, int K,
                                       void* C, int64_t ldc, int out_f32, int bn, jenga_stream_t stream);

/**
 * jenga_test_exp2 -- y_fma[i] = 2^x[i] by the FMA-pipe exponential the scoring kernel uses
 * for part of its columns (cubic on [-1/2, 1/2] after a binary split of x, inputs clamped
 * to [-125, 64]), and y_mufu[i] = 2^x[i] by the hardware approximation (ex2.approx.ftz).
 * x, y_fma, y_mufu: device fp32 arrays of n elements.  For accuracy tests only. */
JENGA_API jenga_status jenga_test_exp2(const float* x, float* y_fma, float* y_mufu, int n, jenga_stream_t stream);

/**
 * jenga_test_wait_timeout -- exercises the device-side wait bound (no counterpart in the
 * paper).  Launches one warp that waits on a shared-memory barrier nothing ever completes;
 * after the current wait budget (jenga_set_wait_budget_ns) it records JENGA_ETIMEOUT (site 8,
 * detail 0xC0FFEE) in the device error word and returns, with nothing else in flight.  The
 * next jenga_check_device_status(stream) then returns JENGA_ETIMEOUT.  Set a short budget
 * first (the default is 2 s) and restore it afterwards.  For tests only. */
JENGA_API jenga_status jenga_test_wait_timeout(jenga_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* JENGA_H_ */
