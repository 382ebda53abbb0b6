/*
 * lq_state.h -- C ABI of the windowed low-bit recurrent-state decode library
 * (liblq.so), for Gated DeltaNet (one decay per head) and KDA (one decay per
 * key channel) on NVIDIA B200 (sm_100a).
 *
 * The operations follow these passages:
 *  - recurrence: "LinQuant: Functional Invariances for Low-Precision Linear
 *    Recurrences", appendix Table 3 (Gated DeltaNet and Kimi Delta Attention
 *    rows).  The state is kept as S (d_k x d_v, key rows, value columns), the
 *    transpose of the table's form:  S_t = (I - b_t k_t k_t^T) D_t S_{t-1}
 *    + b_t k_t v_t^T,  o_t = S_t^T q_t,  D_t = a_t I (GDN) or diag(a_t) (KDA).
 *  - windowed quantization: "LeapQuant: Efficient Linear Attention with
 *    Accurate Recurrent State Quantization" (project page), paragraph on
 *    leaping over a window: the state is stored in low precision at the
 *    window start and held fixed; higher-precision token updates are
 *    buffered; each output comes from the fixed state plus the buffer; at the
 *    window end the full state is reconstructed and quantized again.
 *  - Compensator Tokens: same page, next paragraph: a few high-precision
 *    rank-one outer products keep the largest outliers and share the real
 *    tokens' update path.
 *  - smoothing: same page, following paragraph: per-key-row scales balance
 *    the residual before quantizing, recomputed at every window boundary;
 *    key-row and value-column scales also in "How does STEPQuant compress
 *    recurrent states without losing accuracy?".
 *  - BF16 rows: "DAMP: Decay-Aware Mixed-Precision Recurrent-State
 *    Quantization", abstract: high-risk channels stored at higher precision,
 *    the rest in INT8.
 *
 * Conventions for every call:
 *  - d_* arguments are DEVICE pointers owned by the caller (for instance the
 *    data_ptr() of torch tensors); h_* arguments are HOST pointers.  Nothing
 *    is freed by the library except the opaque handle in lq_state_destroy.
 *  - Floating-point tensors are float32, C-contiguous, in the shapes given.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Compute
 *    calls are asynchronous on it unless their comment says they synchronize.
 *  - Every call returns LQ_OK (0) or a negative lq_status; argument errors are
 *    detected on the host before anything is launched, and a call that
 *    returns an error has launched nothing.  No C++ exception crosses the ABI.
 *  - Supported head sizes: d_k, d_v in {64, 128}.
 */
#ifndef LQ_STATE_H
#define LQ_STATE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LQ_OK = 0,
    LQ_ERR_INVALID_ARG = -1,  /* null pointer, bad enum, W < 1, r > min(dk,dv), ... */
    LQ_ERR_SHAPE = -2,        /* B, H, Hk, dk, dv inconsistent or Hk does not divide H */
    LQ_ERR_WORKSPACE = -3,    /* workspace too small or not 256-byte aligned */
    LQ_ERR_WINDOW_FULL = -4,  /* lq_decode_step with W tokens already buffered */
    LQ_ERR_CUDA = -5,         /* a CUDA runtime call or launch failed */
    LQ_ERR_NONFINITE = -6,    /* a kernel saw a NaN/Inf output (lq_get_status) */
    LQ_ERR_UNSUPPORTED = -7,  /* head size or combination not built */
    LQ_ERR_TIMEOUT = -8       /* a bounded device wait gave up (lq_get_status) */
} lq_status;

typedef enum { LQ_GATE_SCALAR = 0 /* GDN */, LQ_GATE_CHANNEL = 1 /* KDA */ } lq_gate;

typedef enum {
    LQ_MODE_FP32 = 0,        /* FP32 state, read and written every token (baseline) */
    LQ_MODE_INT8_STEP = 1,   /* INT8 state requantized after every token (W must be 1) */
    LQ_MODE_INT8_WINDOW = 2  /* INT8 state quantized once per window of W tokens */
} lq_mode;

/* Longest supported window (tokens buffered between two quantizations). */
#define LQ_MAX_WINDOW 4096

typedef struct {
    int32_t B, H, Hk;       /* batch, value heads, q/k heads (Hk divides H; GQA map h -> h*Hk/H) */
    int32_t dk, dv;         /* key / value head size */
    int32_t gate;           /* lq_gate */
    int32_t mode;           /* lq_mode */
    int32_t W;              /* window length (tokens per quantization), 1 .. LQ_MAX_WINDOW */
    int32_t r;              /* compensator tokens per head, 0..min(dk,dv) */
    int32_t power_iters;    /* power-iteration steps per compensator (K), >= 0 */
    int32_t n_hp_rows;      /* P: BF16 key rows per head (DAMP layout), 0 = all INT8 */
    int32_t smoothing;      /* 1: per-key-row RMS smoothing, column scales from each window's
                               amax; 0: none (m = 1); 2: fixed key-row and value-column scales
                               fitted offline (STEPQuant article; lq_fit_static_scales), given
                               to lq_state_init_static -- INT8 modes, no BF16 rows */
    int32_t fused_flush;    /* 1: the call that buffers the W-th token also flushes */
    int32_t buffer_bf16;    /* 1 (INT8_WINDOW only): keep each buffered token's update in BF16 --
                               bf16(k/Gamma) and bf16(u), formed in FP32, the state carrying the
                               rounded term from that token on (its own output included);
                               compensators stay FP32.  Halves the window buffer's bytes.
                               Not built together with BF16 rows (n_hp_rows > 0:
                               LQ_ERR_UNSUPPORTED).  0: FP32 buffer (the method as stated). */
    int32_t state_bits;     /* code width of the quantized state (INT8 modes and the codec): 8 (0
                               reads as 8), 6 or 4 -- the LeapQuant page's 8-, 6- and 4-bit states:
                               the same quantizer with codes in [-qmax, qmax], qmax = 2^(b-1) - 1
                               (127, 31, 7), s_c = amax_c / qmax.  6 and 4 are bit-packed in the
                               workspace (0.75 and 0.5 bytes a code); views (lq_qstate_view) keep
                               one code per int8 byte.  Not built with BF16 rows (n_hp_rows > 0:
                               LQ_ERR_UNSUPPORTED); FP32 mode takes 0 or 8 only. */
} lq_config;

/* A quantized state in plain arrays (all device pointers, caller-owned):
 *   codes     int8   [B,H,dk-P,dv]  INT8 key rows in increasing row order, dv contiguous
 *                                   (one code per byte also with state_bits 6 or 4)
 *   bf16_rows uint16 [B,H,P,dv]     BF16 bit patterns of the rows listed in hp_row_ids
 *   m         float  [B,H,dk]       smoothing scale per key row (1 on BF16 rows)
 *   s         float  [B,H,dv]       quantization scale per value column
 *   comp_k    float  [B,H,r,dk]     compensator key-side vectors c_j
 *   comp_v    float  [B,H,r,dv]     compensator value-side vectors w_j
 * The represented state is  S_ic = (C_ic * s_c) * m_i  (float, in that order) on
 * INT8 rows, bf16(B_pc) on BF16 rows, plus sum_j c_j[i] w_j[c].
 * bf16_rows may be NULL when P = 0; comp_k/comp_v may be NULL when r = 0. */
typedef struct {
    int8_t *codes;
    uint16_t *bf16_rows;
    float *m;
    float *s;
    float *comp_k;
    float *comp_v;
} lq_qstate_view;

typedef struct lq_state lq_state; /* opaque; host memory owned by the library */

/* Bytes of device workspace lq_state_init needs for cfg (0 if cfg is invalid). */
size_t lq_workspace_bytes(const lq_config *cfg);

/* Check a config without touching the GPU; returns LQ_OK or the error code. */
int lq_config_check(const lq_config *cfg);

/*
 * Create a decode state in caller-owned device memory d_workspace (>=
 * lq_workspace_bytes(cfg) bytes, 256-byte aligned) from an FP32 initial state
 * d_S0 [B,H,dk,dv].  INT8 modes quantize it (compensators, smoothing, codes);
 * FP32 mode copies it.  h_hp_row_ids [H,P] (HOST, required iff P > 0) lists
 * each head's BF16 key rows, distinct and in [0,dk); the same rows serve every
 * batch entry.  Synchronizes `stream` once (status word reset).  The handle
 * must be released with lq_state_destroy; the workspace must outlive it.
 */
int lq_state_init(lq_state **out, const lq_config *cfg, void *d_workspace, size_t bytes,
                  const float *d_S0, const int32_t *h_hp_row_ids, void *stream);

/*
 * lq_state_init for smoothing = 2: the quantizer keeps the given per-head
 * scales at every window boundary -- key rows d_static_m [H,dk] (positive,
 * finite) and value columns d_static_s [H,dv] (>= 0, finite; a zero column
 * quantizes to 0), e.g. from lq_fit_static_scales -- instead of the window's
 * row RMS and column amax; codes beyond +-qmax saturate.  The scales are
 * copied into the workspace (lq_workspace_bytes counts them).  No BF16 rows.
 * Errors as lq_state_init; LQ_ERR_INVALID_ARG for NULL or misaligned scales
 * or smoothing != 2 (and lq_state_init with smoothing = 2).
 */
int lq_state_init_static(lq_state **out, const lq_config *cfg, void *d_workspace, size_t bytes,
                         const float *d_S0, const float *d_static_m, const float *d_static_s, void *stream);

/*
 * Decode one token for all B*H heads:  q, k [B,Hk,dk], v [B,H,dv], beta [B,H],
 * alpha [B,H] (GDN) or [B,H,dk] (KDA)  ->  o [B,H,dv].
 * INT8_WINDOW: the output comes from the window-start INT8 state, its
 * compensators and the buffered updates; the new update (k_t / Gamma_t, u_t)
 * is appended to the buffer and the INT8 state is not written.  Decay guard:
 * Gamma_t (per key channel for KDA) is held as G_t * sigma_t with G_t in
 * [2^-64, 1] keying the buffer and sigma_t a power of two (or 0) scaling the
 * INT8 state; when a decay product would fall below 2^-64 the buffered keys
 * of that channel are rescaled by 2^-64 in place (exact), or zeroed when one
 * token's decay takes it below 2^-128 -- so any decays in [0, 1] and any
 * window length up to LQ_MAX_WINDOW keep the buffered keys finite.  With
 * fused_flush = 1 the call that buffers the W-th token also reconstructs and
 * requantizes the state (the window ends); with fused_flush = 0 a call with W
 * tokens already buffered returns LQ_ERR_WINDOW_FULL and launches nothing.
 * INT8_STEP: decode and requantize in the same launch, every token.
 * FP32: read, update and write the FP32 state.
 */
int lq_decode_step(lq_state *st, const float *d_q, const float *d_k, const float *d_v,
                   const float *d_beta, const float *d_alpha, float *d_o, void *stream);

/*
 * Staggered windows: give every batch entry its own window schedule.  The
 * LeapQuant project page's window paragraph quantizes a sequence's state once
 * every W of its tokens; it does not tie the sequences of a batch to common
 * window ends (in serving they join at different times).  With phases, batch
 * entry b ends a window at the lq_decode_step calls whose index `since`
 * (counted from this call, from the last lq_window_flush, from 0) satisfies
 * (since + h_phase[b]) mod W = W - 1: its first window holds W - h_phase[b]
 * tokens, every later one W.  A step then ends the windows of the entries of
 * one phase only, so the window-end work of 1/W of the batch (phases b mod W)
 * runs beside the buffering of the rest instead of all of it in one step.
 * The window-end launch goes to a higher-priority stream the state owns,
 * forked from `stream` and joined back into it with events before the call
 * returns (stream-ordered: the next call on `stream` sees its results).
 *
 * h_phase [B] (HOST): phases in [0, W); NULL removes the phases (common
 * windows again).  INT8_WINDOW with fused_flush = 1 only, and only while
 * every entry is at a window start (lq_state_buffered = 0): else
 * LQ_ERR_UNSUPPORTED; a phase outside [0, W): LQ_ERR_INVALID_ARG.  Copies the
 * phases into the workspace and synchronizes `stream` once.
 * With phases, entry b holds min((since + h_phase[b]) mod W, since) tokens;
 * lq_window_flush ends every entry's window and restarts the schedule
 * (since = 0); lq_state_buffered returns the most any entry holds;
 * lq_state_export_view and lq_state_import_view need every entry at a window
 * start (LQ_ERR_UNSUPPORTED otherwise) and leave the schedule as it is.
 */
int lq_state_set_phases(lq_state *st, const int32_t *h_phase, void *stream);

/* End the current window: reconstruct S = Gamma (Deq + comps + buffer) and
 * quantize it (new compensators, smoothing, codes); resets the buffer.  A no-op
 * with nothing buffered and in FP32 / INT8_STEP modes. */
int lq_window_flush(lq_state *st, void *stream);

/* Tokens buffered in the current window (host counter, no synchronization);
 * with window phases the most any batch entry holds. */
int lq_state_buffered(const lq_state *st);

/* Write the exact current state, Gamma (Deq + comps + buffer) in INT8 modes or
 * the FP32 state, to d_S [B,H,dk,dv].  Does not change the state. */
int lq_state_export_fp32(const lq_state *st, float *d_S, void *stream);

/* Copy the window-start quantized state out to / in from plain arrays (layout of
 * lq_qstate_view, for this state's B and H).  Import starts a new window
 * (buffer emptied, Gamma = 1); with state_bits 6 or 4 it saturates codes to
 * +-qmax; with smoothing = 2 the imported m and s are the fixed scales from
 * then on.  INT8 modes only.  Used for checkpoint/resume.  Export is taken at
 * a window boundary: with tokens buffered it returns LQ_ERR_UNSUPPORTED (the
 * decay guard of lq_decode_step may have rescaled the stored compensators). */
int lq_state_export_view(const lq_state *st, const lq_qstate_view *out, void *stream);
int lq_state_import_view(lq_state *st, const lq_qstate_view *in, void *stream);

/*
 * Stateless codec on B*H heads.  lq_quantize_state: d_S [B,H,dk,dv] -> out
 * (compensators by power iteration, smoothing, per-column scales, INT8 codes,
 * BF16 rows).  lq_dequantize_state: in -> d_S.  cfg supplies B, H, dk, dv, r,
 * power_iters, smoothing and P; h_hp_row_ids [H,P] is a HOST array (NULL iff
 * P = 0), checked on the host; when P > 0 a device copy of it lives in a
 * stream-ordered temporary (cudaMallocAsync / cudaFreeAsync on `stream`).
 */
int lq_quantize_state(const lq_config *cfg, const float *d_S, const int32_t *h_hp_row_ids,
                      lq_qstate_view *out, void *stream);
int lq_dequantize_state(const lq_config *cfg, const lq_qstate_view *in,
                        const int32_t *h_hp_row_ids, float *d_S, void *stream);

/*
 * lq_quantize_state without any device allocation (the method's pages have no
 * counterpart to this call; it exists for callers of this library).
 *
 * lq_quantize_state keeps the BF16 row list on the device in a temporary it
 * allocates on `stream`.  Some callers cannot let a library allocate: engines
 * whose allocator owns all device memory (it is reserved up front, and an
 * outside cudaMallocAsync would fail or fragment it) and processes that must
 * not allocate after start-up.  This variant is the same computation with the
 * row list held in a fixed array of LQ_STATIC_ROWS_MAX int32 values compiled
 * into the library (a file-scope __device__ array, present on every GPU that
 * loads the library until the process exits).  Same arguments, results and
 * errors as lq_quantize_state, plus:
 *  - LQ_ERR_UNSUPPORTED when H * n_hp_rows > LQ_STATIC_ROWS_MAX;
 *  - the first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture;
 *  - every call copies h_hp_row_ids into the array with cudaMemcpyAsync on
 *    `stream` (from the caller's host memory, read by that copy);
 *  - every call, on every stream, shares the one array and overwrites it:
 *    calls that overlap on the GPU race with each other.
 */
#define LQ_STATIC_ROWS_MAX 8192
int lq_quantize_state_static(const lq_config *cfg, const float *d_S, const int32_t *h_hp_row_ids,
                             lq_qstate_view *out, void *stream);

/*
 * Static scales for smoothing = 2 (offline; STEPQuant article: key-row and
 * value-column scales fitted jointly from the state distribution and each key
 * row's impact on the output error).  Per head h, on the residuals of the
 * n_states calibration states d_states [n_states,H,dk,dv] after cfg->r
 * compensators (K = cfg->power_iters, FP64 extraction), minimise
 *   sum_states sum_i sum_c w_i (R_ic - (clamp(rne((R_ic/m_i)/s_c)) s_c) m_i)^2
 * (codes of cfg->state_bits) over d_m [H,dk] and d_s [H,dv], by 3 rounds of
 * coordinate descent from m_i = RMS of row i over the states (1 if 0), s_c =
 * max |R_ic / m_i| / qmax: each column takes the best of s_c0 (1 - j/16),
 * j = 0..11, then each row the best of m_i0 x {1/2, 5/8, 3/4, 7/8, 1, 5/4,
 * 3/2, 7/4, 2} (first best kept; the objective never increases).  Row weight
 * w_i = each row's impact, read as its decay persistence 1 / (1 - mean decay)
 * (DAMP abstract: decay persistence), from the calibration decays d_gates
 * [n_gate_samples,H,1] (GDN, cfg->gate scalar: one weight per head) or
 * [n_gate_samples,H,dk] (KDA: per key channel), the mean taken in double in
 * sample order; d_gates NULL: w_i = 1.  A stream-ordered temporary of
 * n_states*H*dk*dv floats holds the residuals.  No BF16 rows.
 */
int lq_fit_static_scales(const lq_config *cfg, int32_t n_states, const float *d_states,
                         int32_t n_gate_samples, const float *d_gates, float *d_m, float *d_s, void *stream);

/*
 * Chunked prefill, the step before the windowed decode: T tokens of the
 * recurrence S_t = (I - b k k^T) D_t S_{t-1} + b k v^T, o_t = S_t^T q_t (the
 * rule lq_decode_step follows in FP32 mode; LinQuant appendix Table 3,
 * key-rows form) for all B*H heads, from d_S0 (FP32 [B,H,dk,dv]; NULL = the
 * zero state) to d_S_out [B,H,dk,dv] (may equal d_S0).  Chunks of
 * LQ_PREFILL_CHUNK tokens in WY form: the chunk's rank-one updates become
 * pseudo-values u by forward substitution, with every decay factor
 * 2^(g_t - g_i), i <= t, from cumulative log2 decays (at most 1 for gates in
 * (0, 1]; gates are floored at 2^-150; factors below 2^-126 are flushed to
 * zero).  FP32-level accuracy: the d_k x d_v products run on the tensor cores
 * in three TF32 passes, the rest in FP32.  With dk = dv = 128 and q, k, v
 * (and KDA's alpha) 16-byte aligned the state is held in tensor memory and
 * the inputs arrive by tensor copies; other shapes and alignments take a
 * register-state kernel -- the same results up to rounding order.
 *   inputs, token-major stacks of decode-step inputs: q, k [T,B,Hk,dk],
 *     v [T,B,H,dv], beta [T,B,H], alpha [T,B,H] (GDN) or [T,B,H,dk] (KDA)
 *   d_o [T,B,H,dv] receives every token's output (NULL: not written)
 * cfg supplies B, H, Hk, dk, dv and gate (mode and codec fields unused).
 * T = 0 writes S0 (or zeros) to d_S_out.  To decode from the result with a
 * quantized state, pass d_S_out to lq_state_init, which quantizes it
 * (compensators, smoothing, codes).  Device pointers, caller-owned;
 * asynchronous on `stream`; LQ_ERR_INVALID_ARG for a NULL input with T > 0,
 * T < 0 or T > 2^30, misaligned (not 4-byte) pointers, LQ_ERR_SHAPE / _UNSUPPORTED as
 * for lq_config_check.
 */
#define LQ_PREFILL_CHUNK 16
int lq_prefill(const lq_config *cfg, int32_t T, const float *d_q, const float *d_k, const float *d_v,
               const float *d_beta, const float *d_alpha, const float *d_S0, float *d_S_out, float *d_o,
               void *stream);

/*
 * DAMP channel risk (offline calibration; DAMP abstract: error energy and
 * decay-based persistence pick the high-risk channels).  For each head h:
 *   E[h,i]  = sum_n sum_c (R - Deq(R))_ic^2 over the n_states FP32 states
 *             d_states [n_states,H,dk,dv], R being the residual after cfg->r
 *             compensators and Deq its INT8 reconstruction (no BF16 rows,
 *             smoothing per cfg->smoothing);
 *   score   = E[h,i] / (1 - mean decay), the mean taken over the
 *             n_gate_samples calibration gates d_gates [n_gate_samples,H,ga]
 *             (ga = 1 for GDN: one mean per head; ga = dk for KDA: per row);
 *   d_rows [H,P] <- the P = cfg->n_hp_rows best rows per head (ties to the
 *             lower index) in increasing row order; d_energy [H,dk] <- E.
 * Uses cfg's H, dk, dv, gate, r, power_iters, smoothing, n_hp_rows (>= 1).
 */
int lq_damp_select(const lq_config *cfg, int32_t n_states, const float *d_states,
                   int32_t n_gate_samples, const float *d_gates, double *d_energy,
                   int32_t *d_rows, void *stream);

/*
 * Self-test of the library's internal division (no counterpart in the papers:
 * a check of an implementation detail).  The codec divides by a per-row
 * smoothing scale and a per-column quantization scale many times over; it
 * does so from one correctly rounded reciprocal y = RN(1/b) per divisor and
 * Markstein's FMA correction step, falling back to IEEE division near the
 * subnormal range.  This call runs that routine and the IEEE division on
 * the same operands so that a test can require them to agree bit for bit:
 *   d_fast[i] = the routine's a[i] / b[i];
 *   d_pair[i] = the two-lane variant's a[i] / b[i & ~1] (pairs share b);
 *   d_ieee[i] = IEEE RN a[i] / b[i].
 * All arrays are device arrays of n floats (n even, >= 0); b[i] > 0.
 * Returns LQ_OK, LQ_ERR_INVALID_ARG or LQ_ERR_CUDA.
 */
int lq_selftest_division(const float *d_a, const float *d_b, float *d_fast, float *d_pair, float *d_ieee,
                         int32_t n, void *stream);

/*
 * Self-test of failure detection (not part of the method; no page describes
 * it).  Every staging copy of the decode kernels waits on an mbarrier with a
 * time limit, and a wait that runs out raises the state's timeout status
 * instead of hanging.  This call makes one such wait run out on purpose: one
 * 32-thread block arms an mbarrier for 32 bytes, issues a single 16-byte bulk
 * copy of the state's first workspace bytes (read only), and waits at most
 * limit_ns nanoseconds (1e3 .. 1e9) for a phase that cannot complete; it then
 * raises the timeout bit of this state's status word and returns, waiting a
 * further (bounded) while for nothing.  Afterwards lq_get_status(st) returns
 * LQ_ERR_TIMEOUT (the status is sticky).  Nothing else is written.
 * LQ_ERR_INVALID_ARG for a null state or a limit out of range; LQ_ERR_CUDA
 * if the launch fails.
 */
int lq_selftest_wait(lq_state *st, int64_t limit_ns, void *stream);

/* Synchronize `stream` and return the sticky device status of this state:
 * LQ_OK, LQ_ERR_NONFINITE or LQ_ERR_TIMEOUT. */
int lq_get_status(lq_state *st, void *stream);

void lq_state_destroy(lq_state *st);

const char *lq_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* LQ_STATE_H */
