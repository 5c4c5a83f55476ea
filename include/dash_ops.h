/*
 * dash_ops.h -- building blocks of dash_layer_forward exported for
 * per-kernel parity tests and benchmarks.  Conventions are those of dash.h
 * (device pointers owned by the caller, bf16 bit patterns, row-major,
 * asynchronous on `stream`, host-side argument checks before any launch).
 *
 * Page cited: [DASH blog] "DASH：基于注意力增量的Transformer令牌压缩，实现长序列推理高效加速",
 * §2.1 (the block H -> norm -> attention -> U, H' = H + U, whose pieces these are).
 */
#ifndef DASH_OPS_H_
#define DASH_OPS_H_

#include "dash.h"

#ifdef __cplusplus
extern "C" {
#endif

/* RMSNorm: Y[r] = X[r] * rsqrt(mean(X[r]^2) + eps) * g, fp32 math.
 * X, Y: [M, d] bf16, g: [d].  Requires d % 8 == 0 and d <= 4096. */
dash_status dash_rmsnorm(const dash_bf16* X, int64_t M, int32_t d, const dash_bf16* g, double eps,
                         dash_bf16* Y, void* stream);

/* Y[M, N] = A[M, K] * W[N, K]^T on the tensor cores (tcgen05, fp32
 * accumulation in TMEM, bf16 out).  Requires K % 64 == 0, N % 128 == 0,
 * 16-byte aligned pointers. */
dash_status dash_linear(const dash_bf16* A, int64_t M, int32_t K, const dash_bf16* W, int32_t N,
                        dash_bf16* Y, void* stream);

/* Selects the tile schedule of every tensor-core GEMM launched afterwards by
 * this process (dash_linear and the projections inside the layer and prefill
 * calls).  enable != 0 (the default): GEMMs whose output width splits into
 * 256-column tiles and with more than 128 rows run as 256 x 256 tiles on SM
 * pairs (2-CTA clusters sharing one tcgen05 MMA), when the device can
 * co-schedule them; enable == 0: 128 x 256 / 128 x 128 tiles on single SMs.
 * Both accumulate each output element in fp32 over k in the same order.
 * Returns the previous setting.  Not synchronised with launches in flight on
 * other host threads. */
int32_t dash_set_gemm_pairs(int32_t enable);

/* Selects the form of the generation step's projections (dash_decode_step)
 * for 3 or more sequences: enable != 0 (the default) runs them on the tensor
 * cores (weight rows on the MMA's M dimension, the sequences' rows padded to
 * 16 on N, K split over SMs with a fixed-order reduction) when the shapes
 * suit it (rows a multiple of 128, K of 64); enable == 0: the CUDA-core
 * GEMV.  Both accumulate in fp32; the summation order differs.  Returns the
 * previous setting.  Not synchronised with launches in flight on other host
 * threads. */
int32_t dash_set_decode_tensor_cores(int32_t enable);

/* Causal grouped-query attention (the attention module of §2.1):
 *   Q: [M, hq*hd], K, V: [T_kv, hkv*hd], O: [M, hq*hd] bf16.
 *   Query i sees key j iff kstart(i) <= j <= qpos(i) and j < T_kv, where
 *   qpos(i) = qpos[i] (ascending int32 positions) or i when qpos is NULL,
 *   and kstart(i) = kstart[i] (non-decreasing; the start of row i's own
 *   sequence in a varlen batch, making attention block-diagonal) or 0 when
 *   kstart is NULL.
 *   Scale 1/sqrt(hd), fp32 softmax.  hd must be 64 or 128, hq % hkv == 0. */
dash_status dash_attention(const dash_bf16* Q, const dash_bf16* K, const dash_bf16* V, int64_t M,
                           int64_t T_kv, int32_t hq, int32_t hkv, int32_t hd, const int32_t* qpos,
                           const int32_t* kstart, dash_bf16* O, void* stream);

/* Attention of one new query row per sequence over that sequence's cache
 * (the generation-step attention of dash_decode_step; [DASH blog] §3.1,
 * generation stage):  O[s, h, :] = softmax_j(Q[s, h, :] . k_j / sqrt(hd)) v_j
 * over the rows j < caches[s].len of caches[s] (kv head h / (hq / hkv)).
 *   Q, O: [nseq, hq*hd] bf16; caches: HOST array [nseq] (only k, v, len
 *   are read; 1 <= len <= 2^31 - 1).  nseq <= DASH_DECODE_MAX_SEQ,
 *   hq / hkv <= 16, nseq * hkv <= 64, hd 64 or 128.
 *   ws: dash_decode_attention_workspace_size(hd) bytes. */
size_t dash_decode_attention_workspace_size(int32_t hd);
dash_status dash_decode_attention(const dash_bf16* Q, int32_t nseq, const dash_kv_cache* caches, int32_t hq,
                                  int32_t hkv, int32_t hd, dash_bf16* O, void* ws, size_t ws_bytes,
                                  void* stream);

/* An exponential on the FMA pipe, which the attention softmax takes for one
 * element in 16 in place of MUFU (a compile-time period; no page
 * counterpart; exported so tests can hold it to its error bound): y[i] = 2^x[i] via x = round(x) + f, a cubic in f on [-0.5, 0.5]
 * (max relative error 7.5e-5) and an exponent-field add; inputs below -125
 * are clamped (result ~2e-38).  x, y: [n] fp32 device arrays. */
dash_status dash_exp2_fma(const float* x, int64_t n, float* y, void* stream);

/* Failure-path self test (no page counterpart): launches one kernel whose
 * bounded mbarrier wait can never complete, waits for it and returns what
 * dash_device_error() then reports -- DASH_ERR_TIMEOUT when the bounded wait
 * gave up after its ~2 s limit as designed.  done: [1] int32 device out,
 * 2 when the wait gave up, 1 if it (wrongly) completed.  Synchronises. */
dash_status dash_selftest_wait_timeout(int32_t* done);

/* ------------------------------------------------------ launch timing --
 * Optional CUDA-event timing of every kernel the library launches (off by
 * default; no page counterpart: this is measurement plumbing).  While
 * recording, each launch is bracketed by two events on its own stream. */
typedef enum dash_kernel_kind {
  DASH_K_ROPE_TABLE = 0, DASH_K_RMSNORM = 1, DASH_K_GEMM_QKV = 2, DASH_K_GEMM_KV_HALTED = 3,
  DASH_K_ATTENTION = 4, DASH_K_GEMM_O = 5, DASH_K_SCORE = 6, DASH_K_GEMM_GATE_UP = 7,
  DASH_K_GEMM_DOWN = 8, DASH_K_SELECT = 9, DASH_K_GATHER = 10, DASH_K_SCATTER = 11,
  DASH_K_GEMM = 12, DASH_K_KV_STORE = 13, DASH_K_DEC_GEMV_QKV = 14, DASH_K_DEC_ATTENTION = 15,
  DASH_K_DEC_GEMV_O = 16, DASH_K_DEC_GEMV_GATE_UP = 17, DASH_K_DEC_GEMV_DOWN = 18, DASH_K_COUNT = 19
} dash_kernel_kind;

typedef struct dash_launch_record {
  int32_t kind;     /* dash_kernel_kind */
  int32_t layer;    /* decoder layer, -1 outside the layer loop */
  int64_t m;        /* rows (GEMM M, attention query rows, selection T, decode sequences) */
  int64_t n;        /* GEMM N, attention key rows (decode: cached keys summed over sequences) */
  int64_t k;        /* GEMM K, attention causal (query, key) pairs (decode: CTAs) */
  float ms;         /* device time between the two events */
  int32_t launches; /* kernel launches inside the record (a GEMM whose last wave runs as a
                       separate launch, the selection's passes) */
} dash_launch_record;

/* Starts recording (clears earlier records).  capacity = max launches kept. */
dash_status dash_timing_start(int32_t capacity);
/* Stops recording, synchronises on the recorded events and copies up to
 * cap records to out (host memory).  Returns the number recorded, or -1. */
int32_t dash_timing_stop(dash_launch_record* out, int32_t cap);
/* Static name of a kernel kind. */
const char* dash_kernel_name(int32_t kind);

#ifdef __cplusplus
}
#endif
#endif /* DASH_OPS_H_ */
