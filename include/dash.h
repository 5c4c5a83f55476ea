/*
 * dash.h -- C ABI of the B200 (sm_100a) Delta-Attention Selective Halting
 * (DASH) long-context prefill library, libdash.so.
 *
 * Pages cited (short name -> page title):
 *   [DASH blog]  "DASH：基于注意力增量的Transformer令牌压缩，实现长序列推理高效加速"
 *                §2.1 (U and Δattn_t = ||U_t||_2), §2.3 (single-shot halting
 *                at layer L_s), §3.1 (algorithm steps, top-K, forced first /
 *                last tokens, gather of the active set), §3.3 (pseudocode).
 *   [DASH news]  "DASH：通过注意力动态监测实现长上下文高效预填充", sections
 *                "层间更新动态监测" (threshold) and "选择性停止机制" (halted
 *                tokens keep their KV-cache state).
 *   [DASH abs]   "Stability Implies Redundancy: Delta Attention Selective
 *                Halting for Efficient Long-Context Prefilling" (abstract).
 *
 * Conventions shared by every entry point:
 *   - Every function returns dash_status; DASH_OK (0) on success.
 *   - Argument errors (null pointers, negative or unsupported sizes, a too
 *     small workspace) are detected on the host before anything is launched;
 *     nothing is written then.
 *   - Array pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains them.  Scratch memory comes from the
 *     caller's workspace (size from the matching *_workspace_size call).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; a call returns before the GPU finishes unless
 *     its comment says it synchronises.
 *   - Activations, weights and K/V caches are 16-bit floats (raw bit
 *     patterns, dash_bf16) in the model's format, dash_dims.dtype: bf16 (the
 *     default) or fp16; row-major.  Entry points without a dash_dims
 *     argument take bf16.  Scores are fp32, token indices int32.
 *   - Faults found on the device (a bounded wait that gave up, an index out
 *     of range, a non-finite score) set a sticky device error word instead of
 *     trapping; dash_device_error() reads and clears it.  While it is set,
 *     the library's pipelined kernels return early.
 */
#ifndef DASH_H_
#define DASH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t dash_bf16; /* 16-bit float bit pattern: bf16, or fp16 where dash_dims.dtype says so */

typedef enum dash_status {
  DASH_OK = 0,
  DASH_ERR_INVALID_ARG = 1, /* null pointer, negative size, unknown enum */
  DASH_ERR_SHAPE = 2,       /* a size the kernels do not support */
  DASH_ERR_NONFINITE = 3,   /* a NaN/Inf score, or ||H_t|| = 0 in relative mode */
  DASH_ERR_NO_MEMORY = 4,   /* workspace smaller than *_workspace_size() */
  DASH_ERR_CUDA = 5,        /* a CUDA runtime / driver call failed */
  DASH_ERR_TIMEOUT = 6,     /* a bounded device-side wait gave up */
  DASH_ERR_INDEX = 7        /* an index list entry out of range */
} dash_status;

/* 16-bit float format of a model's activations, weights and K/V caches.
 * Both run on the same tensor-core instructions at the same rate, with fp32
 * accumulation.  bf16 keeps fp32's exponent range with 8 significant bits;
 * fp16 has 11 significant bits (8x less rounding per stored value) but holds
 * magnitudes up to 65504 only.  A value past that range stored as fp16
 * becomes Inf; nothing checks for it, except that a non-finite Δ score is
 * reported as DASH_ERR_NONFINITE. */
typedef enum dash_dtype {
  DASH_DTYPE_BF16 = 0,
  DASH_DTYPE_F16 = 1
} dash_dtype;

/* Decoder-stack dimensions.  Supported: head_dim 64 or 128; d_model and
 * n_heads*head_dim multiples of 128 (d_model <= 4096); ffn_dim a multiple
 * of 64; n_heads a multiple of n_kv_heads. */
typedef struct dash_dims {
  int32_t n_layers;
  int32_t d_model;    /* d */
  int32_t n_heads;    /* query heads hq */
  int32_t n_kv_heads; /* key/value heads hkv */
  int32_t head_dim;   /* hd */
  int32_t ffn_dim;    /* F */
  double rms_eps;     /* RMSNorm epsilon */
  double rope_theta;  /* RoPE base θ (rotate-half pairs (i, i + hd/2)) */
  int32_t dtype;      /* dash_dtype of every 16-bit array the call passes (0 = bf16) */
} dash_dims;

/* Weights of one pre-norm decoder block ([DASH blog] §2.1: norm ->
 * attention -> U, H' = H + U; then norm -> SwiGLU FFN -> residual).
 * All in the model's 16-bit format, row-major [out_features, in_features],
 * no biases. */
typedef struct dash_layer_weights {
  const dash_bf16* attn_norm; /* [d] RMSNorm gain before attention */
  const dash_bf16* w_qkv;     /* [(hq + 2*hkv)*hd, d]: q heads, then k heads, then v heads */
  const dash_bf16* w_o;       /* [d, hq*hd] */
  const dash_bf16* ffn_norm;  /* [d] RMSNorm gain before the FFN */
  const dash_bf16* w_gate;    /* [F, d] */
  const dash_bf16* w_up;      /* [F, d] */
  const dash_bf16* w_down;    /* [d, F] */
} dash_layer_weights;

typedef enum dash_mode {
  DASH_MODE_PRUNE = 0, /* halted tokens leave the sequence ([DASH blog] §3.1) */
  DASH_MODE_HALT = 1,  /* halted tokens stay frozen, their K/V visible ([DASH news]) */
  DASH_MODE_DENSE = 2  /* no halting: every layer on every token */
} dash_mode;

typedef enum dash_select_kind {
  DASH_SELECT_TOPK = 0,     /* top floor(keep_ratio * n) by score ([DASH blog] §3.1) */
  DASH_SELECT_THRESHOLD = 1 /* score >= threshold ([DASH news] "层间更新动态监测") */
} dash_select_kind;

typedef enum dash_score_kind {
  DASH_SCORE_ABS = 0, /* Δ_t = ||U_t||_2 ([DASH blog] §2.1) */
  DASH_SCORE_REL = 1  /* Δ_t = ||U_t||_2 / ||H_t||_2, H = the layer's input residual */
} dash_score_kind;

typedef struct dash_config {
  int32_t halt_layer; /* L_s, 0-based: layers 0..L_s run on all T tokens ([DASH blog] §2.3) */
  int32_t mode;       /* dash_mode */
  int32_t select;     /* dash_select_kind */
  int32_t score;      /* dash_score_kind */
  double keep_ratio;  /* top-k: keep = 1 - ρ */
  float threshold;    /* threshold mode: keep t iff Δ_t >= threshold */
  int32_t keep_first; /* first tokens always kept (0 = none) */
  int32_t keep_last;  /* last tokens always kept (0 = none) */
  /* Consecutive-layer monitoring ([DASH news] "层间更新动态监测": a token is
   * stable when its update stays below the threshold over several
   * consecutive layers).  Δ is taken at the monitor_layers layers ending at
   * halt_layer and combined by maximum, so with threshold selection a token
   * halts iff its Δ is below the threshold in every monitored layer; top-k
   * ranks by the same maximum.  0 or 1 = the halting layer only; at most
   * halt_layer + 1. */
  int32_t monitor_layers;
} dash_config;

/* Human-readable name of a status code (static string). */
const char* dash_status_string(dash_status s);

/* Reads and clears the sticky device error word.  Synchronises the device.
 * Returns DASH_OK, DASH_ERR_TIMEOUT, DASH_ERR_INDEX or DASH_ERR_NONFINITE
 * (the first one found, in that order of priority: TIMEOUT, INDEX, NONFINITE). */
dash_status dash_device_error(void);

/* ---------------------------------------------------------------- score --
 * Δattn per token ([DASH blog] §2.1: Δattn_t = ||U_t||_2; relative form
 * ||U_t||_2 / ||H_t||_2 when relative != 0).
 *   U, H:  [T, d] bf16 (H may be NULL when relative == 0).
 *   delta: [T] fp32 out; sums of squares accumulate in fp32.
 * In relative mode a row with ||H_t|| = 0 yields Inf/NaN and sets the
 * NONFINITE device error.  Requires d % 8 == 0. */
dash_status dash_score(const dash_bf16* U, const dash_bf16* H, int64_t T, int32_t d,
                       int32_t relative, float* delta, void* stream);

/* --------------------------------------------------------------- select --
 * Number of active tokens in top-k mode ([DASH blog] §3.1):
 * |forced| + floor(keep_ratio * (T - |forced|)), forced = the first
 * keep_first and the last keep_last tokens.  Host-only arithmetic in double. */
int64_t dash_topk_count(int64_t T, double keep_ratio, int32_t keep_first, int32_t keep_last);

/* Workspace bytes dash_select needs for T scores: the key histogram, the
 * candidates of the bucket holding the cut (up to T of them, so ties never
 * truncate) and per-chunk counts. */
size_t dash_select_workspace_size(int64_t T);

/* Active-set selection ([DASH blog] §3.1 and the final sort of §3.3;
 * threshold form from [DASH news]).
 *   scores:  [T] fp32.
 *   kind:    DASH_SELECT_TOPK (uses keep_ratio) or DASH_SELECT_THRESHOLD
 *            (uses threshold: keep iff score >= threshold).
 *   Order among scores: larger first; equal scores (+0 and -0 are equal)
 *   go to the lower index.
 *   idx:     [T] int32 out (capacity T): the active indices, ascending,
 *            unique; forced tokens always included.
 *   halted:  [T] int32 out or NULL: the complement, ascending.
 *   count:   [1] int32 device out: number of active tokens, or -3
 *            (= -DASH_ERR_NONFINITE) if any score is NaN/Inf (then idx is
 *            not written and the NONFINITE device error is set).
 *   ws:      dash_select_workspace_size(T) bytes (DASH_ERR_NO_MEMORY if
 *            smaller); may be NULL when T == 0.
 * All SMs take part: one pass over the scores builds a histogram of the
 * keys' top 11 bits, the bucket holding the cut is resolved exactly, and
 * every SM compacts its own chunk of tokens at offsets known from per-chunk
 * counts.  Identical fp32 inputs give bit-identical outputs. */
dash_status dash_select(const float* scores, int64_t T, int32_t kind, double keep_ratio,
                        float threshold, int32_t keep_first, int32_t keep_last,
                        int32_t* idx, int32_t* halted, int32_t* count,
                        void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------ compact/scatter --
 * Gather of the active rows ([DASH blog] §3.1 "复用活跃集合"):
 * Y[i, :] = X[idx[i], :] for i < K.  X: [T, d], Y: [K, d] 16-bit elements
 * (either format: rows are copied bit for bit), d % 8 == 0.
 * An idx entry outside [0, T) sets the INDEX device error; its row is not
 * written. */
dash_status dash_compact(const dash_bf16* X, int64_t T, const int32_t* idx, int64_t K,
                         int32_t d, dash_bf16* Y, void* stream);

/* Inverse of dash_compact: X[idx[i], :] = Y[i, :]; other rows of X unchanged.
 * idx entries must be distinct (ascending lists from dash_select are). */
dash_status dash_scatter(const dash_bf16* Y, const int32_t* idx, int64_t K, int32_t d,
                         dash_bf16* X, int64_t T, void* stream);

/* ---------------------------------------------------------------- layer --
 * Halt-mode context for one compacted layer ([DASH news] "选择性停止机制":
 * halted tokens keep their state and their K/V stay visible, but issue no
 * queries).  The active rows are the layer's H argument, in ascending
 * original-position order.
 *   active_idx: [M] original positions of the active rows (ascending).
 *   halted_idx: [T - M] original positions of the halted rows (ascending).
 *   h_full:     [T, d] hidden states by original position; rows halted_idx
 *               hold the frozen states (only those rows are read).
 * The K/V of halted rows are recomputed from their frozen states with this
 * layer's weights; queries of active rows attend causally, by original
 * position, over all T rows. */
typedef struct dash_halt_ctx {
  const int32_t* active_idx;
  const int32_t* halted_idx;
  const dash_bf16* h_full;
  int64_t T;
} dash_halt_ctx;

/* Workspace bytes for dash_layer_forward on M query rows with T_kv
 * key/value rows (T_kv = M unless halt mode) and positions below max_pos. */
size_t dash_layer_workspace_size(const dash_dims* dims, int64_t M, int64_t T_kv, int64_t max_pos);

/* One pre-norm decoder block in place on H [M, d] ([DASH blog] §2.1).
 *   pos:   [M] int32 RoPE positions of the rows, ascending, < max_pos; NULL
 *          means 0..M-1.  Attention is causal over the rows' order (prune /
 *          dense), or by original position against all T rows (halt).
 *   halt:  NULL, or the halt-mode context (then pos must be
 *          halt->active_idx and max_pos >= halt->T).
 *   delta: [M] fp32 out or NULL: Δ of this layer's attention update U
 *          (U in fp32 before rounding), absolute or relative to ||H_in||.
 * Requires 1 <= M and the dims constraints above. */
dash_status dash_layer_forward(const dash_dims* dims, const dash_layer_weights* w, dash_bf16* H,
                               int64_t M, const int32_t* pos, int64_t max_pos,
                               const dash_halt_ctx* halt, float* delta, int32_t relative,
                               void* ws, size_t ws_bytes, void* stream);

/* The same block as dash_layer_forward, for callers that cannot allocate
 * device memory: code with no allocator of its own (for example a plugin
 * whose host owns every device buffer), or a latency-bound loop that must
 * not call cudaMalloc / cudaFree because they can synchronise the device.
 * The caller still passes every input and output; the scratch that
 * dash_layer_forward takes from a workspace lives instead in one fixed
 * 32 MiB device array inside the library, which each GPU that loads the
 * library holds until the process exits.  No counterpart on the pages: this
 * is a deployment convenience.
 *   - Shapes whose workspace (dash_layer_workspace_size) exceeds 32 MiB are
 *     rejected with DASH_ERR_NO_MEMORY before anything is launched.
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress, which allocates nothing), so the address stays
 *     right after a device reset.  The first call on a device may load the
 *     library's device code there; make that first call before any stream
 *     capture.
 *   - Every call shares the one array and leaves its contents behind; no
 *     part of it needs to start at zero (each call writes every byte it
 *     reads).  Calls whose executions overlap on the GPU (other streams,
 *     other host threads) race on it and must be serialised by the caller.
 *   - Allocates nothing: no cudaMalloc / cudaFree and no allocating library
 *     routine.  Arguments and errors otherwise as dash_layer_forward. */
dash_status dash_layer_forward_noalloc(const dash_dims* dims, const dash_layer_weights* w, dash_bf16* H,
                                       int64_t M, const int32_t* pos, int64_t max_pos,
                                       const dash_halt_ctx* halt, float* delta, int32_t relative,
                                       void* stream);

/* -------------------------------------------------------------- prefill --
 * Workspace bytes for dash_prefill of T tokens under cfg. */
size_t dash_prefill_workspace_size(const dash_dims* dims, int64_t T, const dash_config* cfg);

/* Single-shot DASH prefill ([DASH blog] §2.3 and §3.1; [DASH news]).
 * Layers 0..halt_layer run on all T tokens; the halting layer's attention
 * update gives Δ (fused into its o_proj epilogue); the active set is
 * selected once and reused by every later layer.
 *   layers:    [dims->n_layers] weights.
 *   H:         [T, d] (model format) in: input hidden states; out: prune -> rows
 *              0..K-1 hold the active tokens' final states (rest undefined);
 *              halt / dense -> all T rows (halted rows frozen at the halting
 *              layer's output).
 *   idx_out:   [T] int32 device out or NULL: active indices, ascending.
 *   K_out:     host out or NULL: number of active tokens (T for dense).
 *   delta_out: [T] fp32 device out or NULL: Δ at the halting layer.
 * Synchronises the stream once, after selection, to read K (this is also
 * where NONFINITE is reported).  Output stays on the device. */
dash_status dash_prefill(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* H,
                         int64_t T, const dash_config* cfg, int32_t* idx_out, int64_t* K_out,
                         float* delta_out, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------- varlen prefill --
 * dash_prefill over a batch of independent sequences concatenated along the
 * rows of H ([DASH blog] §5.1: in a batch every sample takes its own halting
 * decision, and gather/scatter must not mix samples).
 *   cu_seqlens: [nseq + 1] HOST int32, cu_seqlens[0] = 0, non-decreasing;
 *               sequence s is rows [cu_seqlens[s], cu_seqlens[s+1]) of H.
 *   Attention is causal within each sequence only (block-diagonal); RoPE
 *   positions count from each sequence's first row; selection (top-k with
 *   K_s = forced + floor(keep * (len_s - forced)), or threshold), forced
 *   first / last tokens and Δ are per sequence.
 *   idx_out:    [T] device out or NULL: active indices (absolute rows),
 *               ascending, grouped by sequence.
 *   seq_counts: [nseq] HOST out or NULL: active tokens per sequence.
 *   Other arguments, output layout and the single synchronisation as in
 *   dash_prefill (prune: the first K rows of H hold the active rows of
 *   sequence 0, then sequence 1, ...). */
size_t dash_prefill_varlen_workspace_size(const dash_dims* dims, int64_t T, int32_t nseq,
                                          const dash_config* cfg);
dash_status dash_prefill_varlen(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* H,
                                const int32_t* cu_seqlens, int32_t nseq, const dash_config* cfg,
                                int32_t* idx_out, int64_t* K_out, int32_t* seq_counts, float* delta_out,
                                void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------ KV cache and generation --
 * [DASH blog] §3.1 (generation stage) and §5.1 (KV cache): generated tokens
 * are not pruned, but the prefill caches keys/values only for the tokens
 * each layer attended over -- in prune mode the active tokens alone in every
 * layer after L_s -- so each generated token attends to fewer keys there.
 *
 * One dash_kv_cache describes one layer of one sequence.  The arrays are
 * caller-owned device memory; `len` is a HOST field the library updates. */
typedef struct dash_kv_cache {
  dash_bf16* k;     /* [capacity, n_kv_heads*head_dim]: keys, RoPE applied, 16-byte aligned */
  dash_bf16* v;     /* [capacity, n_kv_heads*head_dim]: values, 16-byte aligned */
  int32_t* pos;     /* [capacity] original position of each cached row, or NULL */
  int64_t capacity; /* rows allocated */
  int64_t len;      /* rows filled (host field, set by the library) */
} dash_kv_cache;

#define DASH_DECODE_MAX_SEQ 8

/* dash_prefill that also fills caches[0 .. n_layers): layer l's cache gets
 * the keys/values that layer's attention read, in position order, and
 * len = their count:
 *   layers 0..L_s (and every layer in dense mode)  T rows, pos 0..T-1
 *   later layers, prune                            K rows, pos = idx_out
 *   later layers, halt                             T rows (halted rows' keys
 *                                                  from their frozen state)
 * Capacities are checked on the host before any launch (top-k selection),
 * or, with threshold selection, for the later layers right after the
 * selection (DASH_ERR_SHAPE, before those layers run). */
dash_status dash_prefill_kv(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* H, int64_t T,
                            const dash_config* cfg, int32_t* idx_out, int64_t* K_out, float* delta_out,
                            dash_kv_cache* caches, void* ws, size_t ws_bytes, void* stream);

/* dash_prefill_varlen that also fills caches[s * n_layers + l] (sequence-
 * major) for every sequence s, positions counted from the sequence start. */
dash_status dash_prefill_varlen_kv(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* H,
                                   const int32_t* cu_seqlens, int32_t nseq, const dash_config* cfg,
                                   int32_t* idx_out, int64_t* K_out, int32_t* seq_counts, float* delta_out,
                                   dash_kv_cache* caches, void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes for dash_decode_step with up to nseq sequences. */
size_t dash_decode_workspace_size(const dash_dims* dims, int32_t nseq);

/* One generation step: one new token for each of nseq (<= DASH_DECODE_MAX_SEQ)
 * sequences runs through every layer.
 *   X      [nseq, d_model] (model format): the new tokens' input hidden states; on
 *          return the hidden states after the last layer (no final norm).
 *   pos    HOST [nseq]: RoPE position of each new token; it must exceed
 *          every position already in that sequence's cache (the token
 *          attends to all cached rows and itself).
 *   caches HOST array [nseq * n_layers] (sequence-major): each layer appends
 *          the token's key/value (and position) at row len, then len += 1;
 *          every cache needs len < capacity and len + 1 <= 2^31 - 1.
 * Layer l: RMSNorm -> QKV projection with RoPE and the cache append ->
 * attention over the cache -> o_proj + residual -> RMSNorm -> gate/up
 * projection with SwiGLU -> down + residual.  The projections run as
 * CUDA-core GEMVs for 1 or 2 sequences and on the tensor cores for 3 or more
 * when the shapes suit it (dash_set_decode_tensor_cores in dash_ops.h).
 * Requires (n_heads / n_kv_heads) <= 16.  Results are deterministic: a fixed
 * summation order for every sequence count. */
dash_status dash_decode_step(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* X,
                             int32_t nseq, const int32_t* pos, dash_kv_cache* caches, void* ws, size_t ws_bytes,
                             void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DASH_H_ */
