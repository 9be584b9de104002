/*
 * attn_b200.h -- C ABI of the fused attention forward for NVIDIA B200 (sm_100a).
 *
 * One operation:  out = softmax(z + B) V   per (batch n, query head hq, query row i),
 * with the score z in one of two modes and an optional per-head sink logit.
 *
 *   dot   z_ij = scale * <q_i, k_j>
 *         (page "어텐션 메커니즘" section 2, the softmax(QK^T/sqrt(d_k))V definition;
 *          page "SDPA란 무엇인가" section 1, softmax(QK^T/sqrt(E) + B)V and its steps)
 *   rbf   z_ij = -scale * ||q_i - k_j||^2, evaluated in the expanded frame
 *         2*scale*<q_i,k_j> - scale*||k_j||^2 (the query norm cancels by softmax
 *         shift invariance; the key-norm penalty is formed on chip from each key
 *         tile).  (page "Dot-Product Attention을 거리 기반 RBF-Attention으로 교체한
 *          실험기", 섹션별 상세: the squared-distance expansion and the fused kernel)
 *   sink  a per-query-head logit s[hq] joins the softmax denominator but not the
 *         value sum:  out_i = sum_j e^{z_ij} v_j / (e^{s} + sum_j e^{z_ij})
 *         (page "Attention Sink" sections 4.2 and 5.2-5.4)
 *
 * Masks (page "SDPA란 무엇인가" section 1 bias B, section 4 trap 3 alignment;
 * page "어텐션 메커니즘" sections 5 and 6).  With i' = i + (S - L) (bottom-right
 * alignment, so a single decode query sees every cached key):
 *   ATTN_MASK_NONE            every key visible
 *   ATTN_MASK_CAUSAL          key j visible iff j <= i'
 *   ATTN_MASK_SLIDING_WINDOW  key j visible iff 0 <= i' - j < window
 * An additive float bias B[i, j] (0 or -inf; any finite value is added too)
 * composes with every mask kind.  A row with no visible key and no sink yields
 * out = 0 and lse = -inf (SDPA's fully-masked-row convention, page "SDPA란
 * 무엇인가" section 4); with a sink it yields out = 0 and lse = s[hq].
 *
 * Grouped-query attention (page "SDPA란 무엇인가" section 5): query head hq reads
 * KV head hq / (Hq / H).
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { ATTN_DOT = 0, ATTN_RBF = 1, ATTN_SINK = 2 } attn_mode;
typedef enum {
  ATTN_MASK_NONE = 0,
  ATTN_MASK_CAUSAL = 1,
  ATTN_MASK_SLIDING_WINDOW = 2
} attn_mask_kind;
typedef enum { ATTN_BF16 = 0, ATTN_FP32 = 1 } attn_dtype;

/* Status codes.  Every entry point returns ATTN_OK (0) or one of these (< 0). */
typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_NULL_POINTER = -1,   /* q, k, v or out is NULL, or sink is NULL with ATTN_SINK */
  ATTN_ERR_BAD_SHAPE = -2,      /* N, Hq, H, L or S < 1, or a size overflows 64-bit indexing */
  ATTN_ERR_GQA = -3,            /* Hq is not a multiple of H */
  ATTN_ERR_HEAD_DIM = -4,       /* E or Ev not in {64, 128} */
  ATTN_ERR_SCALE = -5,          /* scale not finite or <= 0 */
  ATTN_ERR_MODE = -6,           /* mode out of range */
  ATTN_ERR_MASK = -7,           /* mask_kind out of range */
  ATTN_ERR_WINDOW = -8,         /* window < 1 with ATTN_MASK_SLIDING_WINDOW */
  ATTN_ERR_SINK = -9,           /* ATTN_SINK given without sink logits */
  ATTN_ERR_DTYPE = -10,         /* dtype out of range */
  ATTN_ERR_ALIGNMENT = -11,     /* q, k, v, out or bias not 16-byte aligned; lse not 4-byte aligned */
  ATTN_ERR_WORKSPACE = -12,     /* the library could not allocate its decode workspace */
  ATTN_ERR_CUDA = -13,          /* a CUDA call or kernel launch failed */
  ATTN_ERR_DEVICE_TIMEOUT = -14,/* a kernel gave up a bounded wait (see attn_device_status) */
  ATTN_ERR_DEVICE = -15,        /* the current device is not sm_100 */
  ATTN_ERR_SCRATCH_LIMIT = -16, /* attn_decode_fwd_noalloc: the call needs more scratch than the fixed area holds */
  ATTN_ERR_NOT_DECODE = -17,    /* attn_decode_fwd_noalloc / attn_decode_indexed: not a decode-shaped bf16 call ((Hq/H)*L <= 16) */
  ATTN_ERR_KEEP = -18           /* keep_first < 0 (attn_fwd_streaming, attn_bwd), or kept keys without a window (attn_bwd) */
} attn_status;

/*
 * attn_fwd -- the fused attention forward.
 *
 * Arguments (all pointers are device memory owned by the caller; the library
 * never frees or retains them beyond the call's stream work):
 *   q     [N, Hq, L, E]  contiguous, dtype given by `dtype`
 *   k     [N, H,  S, E]  contiguous
 *   v     [N, H,  S, Ev] contiguous
 *   out   [N, Hq, L, Ev] contiguous, written in the input dtype
 *   lse   [N, Hq, L] float32, natural-log log-sum-exp of each row's logits,
 *         the sink term included (NULL: not written)
 *   scale        > 0; multiplies q.k (dot) or the squared distance (rbf)
 *   mode         ATTN_DOT, ATTN_RBF, or ATTN_SINK (= ATTN_DOT with a required sink).
 *                A non-NULL sink_logits applies the sink in any mode.
 *   sink_logits  [Hq] float32 or NULL
 *   mask_kind    attn_mask_kind; window = number of visible keys per query
 *                (self included) for ATTN_MASK_SLIDING_WINDOW, ignored otherwise
 *   bias         [L, S] float32 additive bias, broadcast over n and heads, or NULL
 *   dtype        ATTN_BF16 (tensor-core path, fp32 accumulation) or ATTN_FP32
 *                (exact fp32 FFMA path)
 *   stream       a cudaStream_t (NULL = the legacy default stream)
 *
 * The call validates every argument first and launches nothing on error.  On
 * success it enqueues its kernels on `stream` and returns without a host
 * synchronisation.  bf16 calls with (Hq/H)*L <= 16 run the split-key decode
 * path (partial kernel + combine kernel), which uses a library-owned device
 * workspace allocated stream-ordered on first need and grown monotonically;
 * all other bf16 calls run the tcgen05 prefill kernel.  With a float bias
 * (outside the streaming mask) a pre-pass first turns the bias into packed
 * keep bits plus per-128-key-tile flags for entries that are neither 0 nor
 * -inf, in the same workspace; flagged tiles add the bias values, so every
 * bias is applied exactly.  Calls on different streams may run concurrently
 * except calls that use the workspace (decode calls and prefill calls with a
 * bias), which must be ordered by the caller.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
             int N, int Hq, int H, int L, int S, int E, int Ev, float scale, int mode,
             const float* sink_logits, int mask_kind, int window, const float* bias,
             int dtype, void* stream);

/*
 * attn_fwd_streaming -- attn_fwd under the StreamingLLM visibility rule: the
 * first keep_first keys (the attention-sink tokens) stay visible to every later
 * query, and otherwise only the last `window` keys are (page "Attention Sink"
 * section 3.2: keep the initial tokens' KV plus a rolling window of recent
 * ones).  With i' = i + (S - L):
 *   key j visible iff  j <= i'  and  (j < keep_first  or  i' - j < window)
 * keep_first = 0 is the sliding window; keep_first >= S is the causal mask.
 *
 * Every other argument, layout, ownership rule, dispatch and status code is
 * attn_fwd's (the mask_kind argument is replaced by window and keep_first).
 * Returns ATTN_ERR_WINDOW for window < 1 and ATTN_ERR_KEEP for keep_first < 0.
 * The kernels read only the key tiles some query of a tile can see: the keys
 * between the kept ones and the window are never loaded.
 */
int attn_fwd_streaming(const void* q, const void* k, const void* v, void* out, float* lse,
                       int N, int Hq, int H, int L, int S, int E, int Ev, float scale, int mode,
                       const float* sink_logits, int window, int keep_first, const float* bias,
                       int dtype, void* stream);

/*
 * attn_bwd -- gradients of attn_fwd's output with respect to q, k, v and the
 * sink logits (bf16 inputs, fp32 gradients).  The sinks and register tokens
 * the pages describe are learned (page "Attention Sink" sections 4.2 and 5;
 * page "Dot-Product Attention을 거리 기반 RBF-Attention으로 교체한 실험기"
 * trains the RBF model), so training needs these.  With P_ij = e^{z_ij - lse_i}
 * on visible keys, D_i = dout_i . out_i and dS_ij = P_ij (dout_i . v_j - D_i):
 *   dv_j = sum_i P_ij dout_i        dq_i = c sum_j dS_ij k_j
 *   dk_j = c sum_i dS_ij q_i  (rbf: minus c k_j sum_i dS_ij)
 *   dsink_h = -sum_{n,i} e^{s_h - lse_i} D_i
 * with c = scale (dot) or 2 scale (rbf).  GQA: dk and dv sum over the query
 * heads of each KV group.
 *
 *   q, k, v     the forward's inputs (bf16, attn_fwd's layouts)
 *   out, lse    the forward's output (bf16 [N, Hq, L, Ev]) and lse (float [N, Hq, L])
 *   dout        bf16 [N, Hq, L, Ev], the loss gradient with respect to out
 *   dq, dk, dv  float outputs, the layouts of q, k, v (caller-owned, overwritten)
 *   dsink       float [Hq] output, or NULL; written when sink_logits is given
 *   scale, mode, sink_logits, mask_kind (NONE, CAUSAL, SLIDING_WINDOW), window:
 *               as in the forward call that produced out and lse
 *   keep_first  0, or with SLIDING_WINDOW the kept initial keys of the
 *               streaming mask (the forward was attn_fwd_streaming)
 *   mask_bits, kv_start, kv_end: the keep bits and key padding of an
 *               attn_fwd_padded forward (each may be NULL)
 * The float bias has no backward here.  Errors: attn_fwd's codes
 * (ATTN_ERR_NULL_POINTER also for out, dout, lse, dq, dk, dv), ATTN_ERR_KEEP
 * for keep_first < 0 or kept keys without SLIDING_WINDOW, ATTN_ERR_ALIGNMENT
 * for mask_bits, kv_start or kv_end not 4-byte aligned.  Uses and grows the
 * library workspace (2*N*Hq*ceil(L/128)*128 floats), so it is ordered with
 * decode calls like they are with each other; no host sync.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
             const float* lse, float* dq, float* dk, float* dv, float* dsink,
             int N, int Hq, int H, int L, int S, int E, int Ev, float scale, int mode,
             const float* sink_logits, int mask_kind, int window, int keep_first,
             const unsigned int* mask_bits, const int* kv_start, const int* kv_end, void* stream);

/*
 * attn_fwd_padded -- attn_fwd with a packed boolean keep mask and per-batch key
 * padding in place of the float bias (page "SDPA란 무엇인가" §1: B holds 0 or
 * -inf; §4 trap 1: in a boolean attn_mask, True marks a pair that takes part;
 * the page's left-padding check: with the mask passed, padded and unpadded
 * inputs give the same output on the real tokens).
 *
 *   mask_bits  [L, ceil(S/32)] uint32, device, or NULL (every pair kept): bit
 *              j % 32 of word i*ceil(S/32) + j/32 set means query row i may
 *              attend to key j.  Broadcast over batch and heads.  32x fewer
 *              bytes than the equivalent float bias.
 *   kv_start   [N] int32, device, or NULL (0): keys j < kv_start[n] are padding
 *              for batch n (left padding).
 *   kv_end     [N] int32, device, or NULL (S): keys j >= kv_end[n] are padding
 *              (right padding / variable length).  Values are clamped to
 *              [0, S]; kv_start >= kv_end leaves batch n no key.
 *
 * Key j is visible to row i of batch n iff the mask kind allows it, its bit is
 * set, and kv_start[n] <= j < kv_end[n].  A row with no visible key gets out = 0
 * and lse = -inf (lse = s with a sink), as SDPA does for left-padded start rows.
 * Tiles of keys wholly inside the padding are not read.  All other arguments,
 * layouts, ownership, dispatch and status codes are attn_fwd's (mask_kind is
 * NONE, CAUSAL or SLIDING_WINDOW); mask_bits, kv_start and kv_end must be
 * 4-byte aligned (ATTN_ERR_ALIGNMENT).
 */
int attn_fwd_padded(const void* q, const void* k, const void* v, void* out, float* lse,
                    int N, int Hq, int H, int L, int S, int E, int Ev, float scale, int mode,
                    const float* sink_logits, int mask_kind, int window,
                    const unsigned int* mask_bits, const int* kv_start, const int* kv_end,
                    int dtype, void* stream);

/*
 * attn_decode_indexed -- exact decode attention over a listed subset of the
 * cached keys: the step that follows a top-k key selection (page "기술 요약:
 * SOCKET - 희소 어텐션을 위한 SOft Collision Kernel EsTimator", 방법론, 핵심
 * 메커니즘 step 4: the top-k keys are chosen, then exact attention is computed
 * on that subset).  The selection itself is the caller's.
 *
 *   key_idx  [N, H, n_sel] int32, device memory owned by the caller: the key
 *            positions (rows of k and v) each (batch, KV head) attends to.  One
 *            list serves all Hq/H query heads of the KV group and all L query
 *            rows.  Entries outside [0, S) (such as -1 padding) select nothing.
 *            A position listed twice counts twice (attention over the gathered
 *            list).  Order does not matter.
 *   n_sel    >= 1, entries per list.
 *
 * The softmax and the value sum run over the listed keys only:
 *   out_i = sum_{j in list} e^{z_ij} v_j / (e^{s} [sink] + sum_{j in list} e^{z_ij})
 * with z_ij = scale * <q_i, k_j>.  mask_kind (NONE, CAUSAL, SLIDING_WINDOW with
 * window), bias [L, S] and the sink are those of attn_fwd, applied at each
 * key's original position j.  A row that sees no listed key gets out = 0 and
 * lse = -inf (lse = s with a sink).
 *
 * q, k, v, out, lse: attn_fwd's layouts, bf16 only (dot score).  The call must
 * be decode-shaped, (Hq/H)*L <= 16, else ATTN_ERR_NOT_DECODE.  Errors: attn_fwd's
 * codes, plus ATTN_ERR_NULL_POINTER for a NULL key_idx, ATTN_ERR_BAD_SHAPE for
 * n_sel < 1, ATTN_ERR_ALIGNMENT for a key_idx not 4-byte aligned.  It uses and
 * grows the same library workspace as attn_fwd's decode path (ordering rules
 * as there) and returns without a host synchronisation.
 */
int attn_decode_indexed(const void* q, const void* k, const void* v, void* out, float* lse,
                        const int* key_idx, int n_sel,
                        int N, int Hq, int H, int L, int S, int E, int Ev, float scale,
                        const float* sink_logits, int mask_kind, int window, const float* bias,
                        void* stream);

/* Human-readable text for a status code (static storage, never NULL). */
const char* attn_status_string(int status);

/* Frees the decode workspace (synchronises the device first).  The next decode
 * call allocates it again. */
void attn_release_workspace(void);

/*
 * attn_device_status -- synchronises `stream`, then reads and clears the
 * device-side status word.  Every wait inside the kernels (on a TMA transfer,
 * a tensor-core commit or a sibling warp) is bounded; a wait that runs out
 * makes its CTA record the fault here, drain its own in-flight copies and
 * tensor-core work, release its tensor memory and exit.  Returns ATTN_OK,
 * ATTN_ERR_DEVICE_TIMEOUT, or ATTN_ERR_CUDA if the synchronisation failed.
 */
int attn_device_status(void* stream);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int attn_version(void);

/*
 * Failure-path checks.  The attention pages have no counterpart to these two
 * functions; they let a test drive the library's error paths without faulting
 * or hanging a GPU.
 *
 * attn_test_wait_timeout -- launches on `stream` one thread that waits on a
 * shared-memory barrier nothing ever arrives at, with a bounded wait of
 * limit_cycles (>= 1) SM clock cycles.  The wait runs out, the thread records
 * the timeout in the device status word as the pipeline kernels' bounded waits
 * do, and the kernel returns; the next attn_device_status reports
 * ATTN_ERR_DEVICE_TIMEOUT once and the context stays usable.  Returns
 * ATTN_OK once launched, ATTN_ERR_BAD_SHAPE for limit_cycles < 1, or
 * attn_fwd's device errors.
 */
int attn_test_wait_timeout(int limit_cycles, void* stream);

/*
 * attn_test_fail_workspace_allocs -- the next `count` (>= 0) allocations of the
 * library workspace (the decode partials, a float bias's keep bits, the
 * backward's per-row terms) fail as a failed cudaMallocAsync would: the call
 * returns ATTN_ERR_WORKSPACE and launches nothing.  A workspace already large
 * enough is not reallocated and does not fail.  0 clears the injection.
 * Returns ATTN_OK, or ATTN_ERR_BAD_SHAPE for count < 0.
 */
int attn_test_fail_workspace_allocs(int count);

/*
 * attn_exp2_poly_eval -- verification hook: y[i] = the prefill softmax's
 * software base-2 exponential of x[i] (device pointers, n floats).  A share of
 * the softmax exponentials is evaluated this way on the FMA pipe instead of
 * the MUFU unit: 2^x = 2^round(x) * p(x - round(x)) with a degree-3 minimax
 * polynomial (relative error <= 1.02e-4); x is clamped to >= -126.  The
 * exponential itself is the softmax's (page "어텐션 메커니즘" §2, §6); this
 * way of evaluating it is an implementation choice, not from the pages.
 */
int attn_exp2_poly_eval(const float* x, float* y, int n, void* stream);

/*
 * attn_decode_fwd_noalloc -- the decode path of attn_fwd (bf16, dot or RBF
 * score, (Hq/H)*L <= 16) without any device allocation.  The attention pages have
 * no counterpart to this entry point; it exists for callers that must not
 * allocate device memory while they run: services that reserve all GPU memory
 * at start-up and forbid later allocations (so latency stays predictable and
 * no out-of-memory error can happen mid-request), and host frameworks whose
 * own allocator owns all device memory.
 *
 * Arguments, layouts, ownership and masks are those of attn_fwd (the dtype is
 * bf16).  Instead of the library's allocated workspace, the partial results
 * live in a fixed scratch array compiled into the library
 * (attn_decode_noalloc_scratch_bytes() bytes, 8 MiB).  The array becomes
 * resident on a device when the library's device code is loaded into that
 * device's context: under CUDA's default lazy module loading that is the first
 * call on the device, which therefore takes the array's 8 MiB and the code's
 * memory once.  Make that first call during start-up, before reserving the
 * rest of the device's memory and before beginning any stream capture (or set
 * CUDA_MODULE_LOADING=EAGER, which loads both with the context).  The array
 * then stays until the context is destroyed.  The first call in a context
 * also looks up the array's device address (cudaGetSymbolAddress) with the
 * device current; a call that finds a different context current (after
 * cudaDeviceReset, say) looks it up again, and that call is again a first
 * call in the sense above.
 * Calls that need more scratch than the array holds return
 * ATTN_ERR_SCRATCH_LIMIT; calls that are not decode-shaped return
 * ATTN_ERR_NOT_DECODE; neither launches anything.  Beyond that module load,
 * the function calls no cudaMalloc, cudaFree or other allocating routine.  All calls share the one
 * array: calls that overlap on the GPU race and must be ordered by the
 * caller.  Nothing in the array needs clearing between calls.
 */
int attn_decode_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                            int N, int Hq, int H, int L, int S, int E, int Ev, float scale, int mode,
                            const float* sink_logits, int mask_kind, int window, const float* bias,
                            void* stream);

/* Size in bytes of the fixed scratch array used by attn_decode_fwd_noalloc. */
size_t attn_decode_noalloc_scratch_bytes(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
