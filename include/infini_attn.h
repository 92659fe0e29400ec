/*
 * infini_attn.h — C ABI of the B200 (sm_100a) Infini-attention forward library.
 *
 * The operation is the Infini-attention layer of "Leave No Context Behind:
 * Efficient Infinite Context Transformers with Infini-attention" (Munkhdalai,
 * Faruqui, Golovnev; arXiv 2404.07143), as quoted on the close-reading note
 * llm-papers-study.pages.dev ("精读笔记：Infini-attention"), section 3.
 * For every (batch b, head h) the sequence of L tokens is cut into segments of N
 * tokens (the last one may be shorter). For segment s, with sigma = ELU + 1 and
 * g_h = sigmoid(beta_h):
 *
 *   A_dot = softmax(Q_s K_s^T / sqrt(d) + causal mask) V_s          (section 3.1)
 *   A_mem = sigma(Q_s) M_{s-1} / (sigma(Q_s) z_{s-1})                 (section 3.3)
 *   out_s = g_h * A_mem + (1 - g_h) * A_dot                           (section 3.5)
 *   Linear:       M_s = M_{s-1} + sigma(K_s)^T V_s                    (section 3.4)
 *   Linear+Delta: M_s = M_{s-1} + sigma(K_s)^T (V_s - sigma(K_s) M_{s-1}
 *                                                 / (sigma(K_s) z_{s-1}))
 *   both modes:   z_s = z_{s-1} + sum_t sigma(K_{s,t})
 *
 * The output of a segment is formed from the state before that segment's update
 * (read, then write: section 3.8 summary; waylandz.com chapter 24, section 24.5).
 * Conventions fixed by this library: the softmax scale is 1/sqrt(d); the causal
 * mask is inside the segment and includes the diagonal; a row whose denominator
 * sigma(x) . z is exactly 0 (the zero state, e.g. the first segment from
 * M_0 = 0, z_0 = 0) retrieves 0 and contributes no delta term; the gate is still
 * applied to such rows.
 *
 * Layouts (all contiguous, row-major):
 *   q, k, v, out : [B, H, L, d]     (bf16 for the plain names, fp32 for *_f32)
 *   beta         : [H] fp32         one gate logit per head, shared by the batch
 *   M            : [B, H, d, d] fp32, row = key feature, column = value feature
 *   z            : [B, H, d] fp32
 *
 * Pointers are device pointers owned by the caller; the library keeps none of
 * them after the call returns. M_in/z_in may be NULL (zero state, both must be
 * NULL together). M_out/z_out may be NULL (state not written; both together) and
 * may equal M_in/z_in (in-place carry: the library reads the old state before it
 * writes the new one). out must not overlap q, k, v, M or z.
 *
 * Execution: every call is asynchronous on `stream` (a cudaStream_t, NULL = the
 * legacy default stream). The return value reports argument errors (checked on
 * the host before any launch) and launch errors. Faults during execution surface
 * at the caller's next synchronisation. No call synchronises with the host and
 * none falls back to the CPU.
 */
#ifndef INFINI_ATTN_H
#define INFINI_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  INFINI_LINEAR = 0, /* section 3.4, Linear update */
  INFINI_DELTA = 1   /* section 3.4, Linear + Delta update */
} infini_mode_t;

typedef enum {
  INFINI_OK = 0,
  INFINI_ERR_NULL = -1,        /* a required pointer is NULL, or M/z NULL-ness mismatched */
  INFINI_ERR_SHAPE = -2,       /* B, H, N < 1, L < 0, or a size product overflows */
  INFINI_ERR_UNSUPPORTED = -3, /* d or mode not supported by this entry point */
  INFINI_ERR_ALIGN = -4,       /* q, k, v or out not 16-byte aligned */
  INFINI_ERR_CUDA = -5,        /* a CUDA runtime call or a launch failed */
  INFINI_ERR_NOMEM = -6,       /* the stream-ordered scratch allocation failed */
  INFINI_ERR_TIMEOUT = -7,     /* a bounded device wait ran out (infini_attn_device_status) */
  INFINI_ERR_ALIAS = -8,       /* out overlaps an input or the state */
  INFINI_ERR_SCRATCH_LIMIT = -9 /* infini_attn_step_static: sizes need more than its fixed scratch */
} infini_status_t;

/*
 * Whole-sequence forward, bf16 q/k/v/out (__nv_bfloat16), fp32 beta/M/z.
 * Requires d == 128. L may be 0 (the state is passed through) and need not be a
 * multiple of N (the last segment is shorter). Scratch memory for the per-segment
 * states is taken from the stream-ordered allocator on `stream` and returned on
 * the same stream before the call returns (INFINI_ERR_NOMEM if that fails).
 */
int infini_attn_forward(const void* q, const void* k, const void* v, const float* beta,
                        const float* M_in, const float* z_in, void* out, float* M_out,
                        float* z_out, int B, int H, long long L, int N, int d, int mode,
                        void* stream);

/*
 * One segment of a stream with carried state (section 3.4: the new state is
 * passed to the next segment). Same as infini_attn_forward with L == N; the
 * output uses (M_in, z_in), then the state advances to (M_out, z_out), which may
 * be the same buffers. bf16 q/k/v/out [B, H, N, d].
 */
int infini_attn_step(const void* q, const void* k, const void* v, const float* beta,
                     const float* M_in, const float* z_in, void* out, float* M_out,
                     float* z_out, int B, int H, int N, int d, int mode, void* stream);

/*
 * infini_attn_step without any device-memory allocation. The paper has no
 * counterpart to this call; it exists for callers that must not allocate on
 * their hot path: a serving loop that reserved its whole memory budget at
 * start-up, or a framework whose own allocator owns all device memory (an
 * allocation made behind its back sits outside its accounting and can fail or
 * fragment). Arguments, layouts and results are those of infini_attn_step
 * (bf16, d == 128); the caller still passes every input and output.
 * Scratch: one fixed 8 MiB array per device, reserved for the life of the
 * process on every GPU that loads the library. Sizes whose scratch does not fit
 * (roughly B*H above 40 heads for one segment) return INFINI_ERR_SCRATCH_LIMIT
 * before any launch. The first call on a device looks up the array's address
 * for that device; make that first call before any stream capture begins. All
 * calls on a device share the array: calls whose GPU work may overlap in time
 * race on it, so order them on one stream or synchronise between them.
 */
int infini_attn_step_static(const void* q, const void* k, const void* v, const float* beta,
                            const float* M_in, const float* z_in, void* out, float* M_out,
                            float* z_out, int B, int H, int N, int d, int mode, void* stream);

/* Memory layouts of q, k, v and out for infini_attn_forward_gqa. */
typedef enum {
  INFINI_LAYOUT_BHLD = 0, /* [B, H, L, d] contiguous (every other entry point) */
  INFINI_LAYOUT_BLHD = 1  /* [B, L, H, d] contiguous: the rows of a [B, L, H * d] projection */
} infini_layout_t;

/*
 * infini_attn_forward with grouped key/value heads and a choice of layout (bf16,
 * d == 128). q and out have H heads, k and v have H_kv heads (H % H_kv == 0); query
 * head h reads key/value head h / (H / H_kv) for its local attention and retrieves
 * from that head's memory, so M and z are [B, H_kv, d, d] and [B, H_kv, d] (the
 * memory is built from K and V only, section 3.4). With H_kv == H and
 * INFINI_LAYOUT_BHLD this is infini_attn_forward. The layout applies to all four of
 * q, k, v, out: [B, H or H_kv, L, d] or [B, L, H or H_kv, d]. beta has H entries.
 * Errors: INFINI_ERR_SHAPE for H_kv < 1 or H % H_kv != 0, INFINI_ERR_UNSUPPORTED for
 * an unknown layout or d != 128; otherwise as infini_attn_forward.
 */
int infini_attn_forward_gqa(const void* q, const void* k, const void* v, const float* beta,
                            const float* M_in, const float* z_in, void* out, float* M_out,
                            float* z_out, int B, int H, int H_kv, long long L, int N, int d,
                            int mode, int layout, void* stream);

/*
 * The memory update alone (section 3.4, Linear or Linear+Delta, applied segment by
 * segment): (M_out, z_out) after L tokens of bf16 k, v [B, H, L, d] cut into
 * segments of N (the last may be shorter), starting from (M_in, z_in) (NULL: the
 * zero state); no attention outputs. For Linear the result is M_in + sum over
 * segments of sigma(K_s)^T V_s and z_in + sum of sigma(K_s) rows, so a sequence split
 * into consecutive ranges can be processed range by range, or on several GPUs: each
 * range's sum from the zero state, an all-gather, and every range's forward from the
 * sum of the ranges before it. Requires d == 128; M_out, z_out required (they may
 * be M_in, z_in); 16-byte aligned k, v, M_in, M_out; the state must not overlap k, v.
 * Scratch from the stream-ordered allocator on `stream` (INFINI_ERR_NOMEM).
 */
int infini_attn_state_update(const void* k, const void* v, const float* M_in, const float* z_in,
                             float* M_out, float* z_out, int B, int H, long long L, int N, int d,
                             int mode, void* stream);

/*
 * (M_out, z_out) = (M_in, z_in) + the sum of `count` state blocks dM [count, B, H, d, d]
 * and dz [count, B, H, d] (fp32, device), added in block order (deterministic).
 * M_in / z_in NULL: the zero state; count may be 0. With infini_attn_state_update this
 * composes Linear-mode states of consecutive ranges of a sequence (section 3.4: the
 * Linear memory is a plain sum over segments). M_out, z_out must not overlap the
 * blocks (they may be M_in, z_in).
 */
int infini_attn_state_sum(const float* dM, const float* dz, int count, const float* M_in,
                          const float* z_in, float* M_out, float* z_out, int B, int H, int d,
                          void* stream);

/*
 * Token-level streaming decode (the pages' "fast streaming inference": section 3.1
 * attention and section 3.3 retrieval for tokens that arrive one or a few at a
 * time inside a segment). n new tokens of every (b, h) join the current segment,
 * whose first `pos` tokens the caller's KV cache already holds.
 *   q, k, v            [B, H, n, d] bf16, the new tokens (device, read).
 *   beta               [H] fp32 (device, read).
 *   k_cache, v_cache   [B, H, N, d] bf16, the current segment's keys and values
 *                      (device, caller-owned): rows [0, pos) are read, rows
 *                      [pos, pos + n) are written with k and v by this call.
 *   M, z               [B, H, d, d] and [B, H, d] fp32 (device): the memory of the
 *                      segments before this one (M_{s-1}, z_{s-1}; zeros at the start
 *                      of a stream). Read for the retrieval; when pos + n == N the
 *                      call then folds the completed segment in with the Linear or
 *                      Linear+Delta rule, in place, so the next call starts the next
 *                      segment with pos = 0.
 *   out                [B, H, n, d] bf16 (device, written): for new token i (segment
 *                      position t = pos + i), g A_mem + (1 - g) A_dot with A_dot the
 *                      causal softmax attention over cache rows 0..t and A_mem the
 *                      retrieval from (M, z) as passed in. Every token gets what
 *                      infini_attn_forward gives it on the same stream of tokens.
 * Requires d == 128, n >= 1, pos >= 0, pos + n <= N, B * H <= 65535, n <= 1048560
 * (65535 groups of 16 tokens), mode 0 or 1, 16-byte aligned pointers and no overlap
 * between out, the caches, the state and the inputs (INFINI_ERR_NULL / SHAPE /
 * UNSUPPORTED / ALIGN / ALIAS before any launch).
 * Scratch comes from the stream-ordered allocator on `stream` (INFINI_ERR_NOMEM).
 * Built for small n; a whole segment at once is cheaper through infini_attn_step.
 */
int infini_attn_decode(const void* q, const void* k, const void* v, const float* beta,
                       void* k_cache, void* v_cache, float* M, float* z, void* out, int B, int H,
                       int n, int pos, int N, int d, int mode, void* stream);

/*
 * Gradient of infini_attn_forward (bf16) with respect to q, k, v, beta and the
 * incoming state, for the loss sum(dout * out) + sum(dM_out * M_out) +
 * sum(dz_out * z_out). The pages define only the forward ("Leave No Context
 * Behind", arXiv 2404.07143, sections 3.1, 3.3-3.5 as quoted on
 * llm-papers-study.pages.dev); this is the chain rule through its steps. A row whose
 * retrieval denominator is exactly 0 (the zero state) retrieves the constant 0 and
 * passes no gradient; sigma'(x) = 1 for x > 0, e^x otherwise.
 *
 *   q, k, v, dout      device, bf16 [B, H, L, d] contiguous, the forward's inputs and
 *                      the gradient of its output
 *   beta               device, fp32 [H]
 *   M_in, z_in         device, fp32 [B, H, d, d] / [B, H, d], the forward's incoming
 *                      state (both NULL: the zero state)
 *   dM_out, dz_out     device, fp32, gradients of the forward's final state (both
 *                      NULL: zero)
 *   dq, dk, dv         device, bf16 [B, H, L, d], written
 *   dbeta              device, fp32 [H], written (summed over the batch)
 *   dM_in, dz_in       device, fp32, gradients of the incoming state (both NULL: not
 *                      written)
 * Requires d = 128, N a multiple of 128 and L a multiple of N
 * (INFINI_ERR_UNSUPPORTED otherwise); every pointer 16-byte aligned; no output may
 * overlap an input or another output (INFINI_ERR_ALIAS). L = 0 writes dbeta = 0 and
 * passes (dM_out, dz_out) through to (dM_in, dz_in). Asynchronous on `stream`;
 * scratch (infini_attn_backward_workspace_size: about 0.6 to 1.1 KB per token and
 * head, mostly per-tile partials of the state gradients) comes from the
 * stream-ordered allocator (INFINI_ERR_NOMEM). The forward's state path runs again
 * inside the call to rebuild every segment's incoming state. Results are bitwise
 * reproducible (every reduction runs in a fixed order).
 */
int infini_attn_backward(const void* q, const void* k, const void* v, const float* beta,
                         const float* M_in, const float* z_in, const void* dout,
                         const float* dM_out, const float* dz_out, void* dq, void* dk, void* dv,
                         float* dbeta, float* dM_in, float* dz_in, int B, int H, long long L,
                         int N, int d, int mode, void* stream);

/*
 * One attention layer with its projections ("Leave No Context Behind", sections 3.1
 * and 3.6 as quoted on llm-papers-study.pages.dev): Q = x W_Q, K = x W_K, V = x W_V
 * (heads side by side in the columns: head h is columns [h d, h d + d)), the
 * grouped-head forward of infini_attn_forward_gqa on them in place ([B, L, heads, d]),
 * then y = [A_1 ... A_H] W_O.
 *   x        device, bf16 [B, L, D_model] row-major
 *   Wq       device, bf16 [D_model, H * d];  Wk, Wv: [D_model, H_kv * d]
 *   Wo       device, bf16 [H * d, D_model]
 *   beta     device, fp32 [H]; M_in/z_in, M_out/z_out as infini_attn_forward_gqa
 *            (per key/value head: [B, H_kv, d, d] and [B, H_kv, d])
 *   y        device, bf16 [B, L, D_model], written
 * Requires d = 128, D_model a multiple of 128 and B * L a multiple of 128
 * (INFINI_ERR_UNSUPPORTED otherwise), H a multiple of H_kv, 16-byte alignment; y may
 * not overlap x or a weight. Asynchronous on `stream`; the projections' outputs
 * (2 (H + H_kv) d bf16 per token) and the forward's scratch come from the
 * stream-ordered allocator.
 */
int infini_attn_layer_forward(const void* x, const void* Wq, const void* Wk, const void* Wv,
                              const void* Wo, const float* beta, const float* M_in,
                              const float* z_in, void* y, float* M_out, float* z_out, int B,
                              long long L, int D_model, int H, int H_kv, int N, int d, int mode,
                              void* stream);

/*
 * C [M][N] = A [M][K] B [K][N]: bf16 row-major in and out, fp32 accumulation on the
 * tensor cores (the layer's projection GEMM). M, N, K multiples of 128
 * (INFINI_ERR_UNSUPPORTED otherwise), M < 2^31 (INFINI_ERR_SHAPE); device pointers,
 * 16-byte aligned; C may not
 * overlap A or B. Asynchronous on `stream`, no scratch.
 */
int infini_attn_gemm_bf16(const void* A, const void* B, void* C, long long M, int N, int K,
                          void* stream);

/* fp32 q/k/v/out variants of infini_attn_forward and infini_attn_step; 1 <= d <= 128,
 * B * H <= 65535 (INFINI_ERR_SHAPE beyond). */
int infini_attn_forward_f32(const float* q, const float* k, const float* v, const float* beta,
                            const float* M_in, const float* z_in, float* out, float* M_out,
                            float* z_out, int B, int H, long long L, int N, int d, int mode,
                            void* stream);
int infini_attn_step_f32(const float* q, const float* k, const float* v, const float* beta,
                         const float* M_in, const float* z_in, float* out, float* M_out,
                         float* z_out, int B, int H, int N, int d, int mode, void* stream);

/*
 * Options for the extended forward. All fields may be zero.
 *   workspace / workspace_bytes: caller-owned device scratch of at least
 *     infini_attn_workspace_size(...) bytes, 256-byte aligned; when NULL the
 *     library uses the stream-ordered allocator as infini_attn_forward does.
 *   stage_events[0..2]: cudaEvent_t handles (or NULL) recorded on `stream`
 *     before the state kernels, between the state kernels and the fused
 *     attention kernel, and after the fused attention kernel. When the call
 *     holds a single segment (L <= N), the attention reads only the incoming
 *     state and the state update runs beside it on a second stream of the
 *     library (forked from and joined back into `stream` within the call):
 *     event 1 then marks the fork, event 2 the point where both are done.
 *     That second stream is one per device for the whole process: one-segment
 *     calls from several host threads take turns on it (a mutex keeps each
 *     fork..join sequence whole), so their state updates run one after another.
 */
typedef struct {
  void* workspace;
  size_t workspace_bytes;
  void* stage_events[3];
} infini_attn_opts_t;

/* dtype codes for the extended calls */
#define INFINI_DTYPE_BF16 0
#define INFINI_DTYPE_F32 1

/* Scratch bytes the forward needs for these sizes (0 when none is needed). */
size_t infini_attn_workspace_size(int B, int H, long long L, int N, int d, int mode,
                                  int dtype);

/* infini_attn_forward / _f32 with options (dtype selects the element type). */
int infini_attn_forward_ex(const void* q, const void* k, const void* v, const float* beta,
                           const float* M_in, const float* z_in, void* out, float* M_out,
                           float* z_out, int B, int H, long long L, int N, int d, int mode,
                           int dtype, const infini_attn_opts_t* opts, void* stream);

/*
 * infini_attn_layer_forward with options: opts->workspace (256-byte aligned, at least
 * infini_attn_layer_workspace_size(...) bytes) holds the projections' outputs and the
 * forward's scratch instead of the stream-ordered allocator; opts->stage_events[0..2]
 * (cudaEvent_t or NULL) are recorded after the Q/K/V projections, after the forward
 * and after the output projection.
 */
int infini_attn_layer_forward_ex(const void* x, const void* Wq, const void* Wk, const void* Wv,
                                 const void* Wo, const float* beta, const float* M_in,
                                 const float* z_in, void* y, float* M_out, float* z_out, int B,
                                 long long L, int D_model, int H, int H_kv, int N, int d, int mode,
                                 const infini_attn_opts_t* opts, void* stream);

/* Scratch bytes infini_attn_layer_forward needs (0 when the sizes are not supported). */
size_t infini_attn_layer_workspace_size(int B, long long L, int D_model, int H, int H_kv, int N,
                                        int d, int mode);

/*
 * infini_attn_backward with options: opts->workspace (256-byte aligned, at least
 * infini_attn_backward_workspace_size(...) bytes) replaces the stream-ordered
 * allocation; opts->stage_events[0..2] (cudaEvent_t or NULL) are recorded on
 * `stream` after the state rebuild, after the dq kernel (which also runs the
 * retrieval's backward) and after the dk/dv kernel (preceded by the reverse state
 * chain; it also runs the memory update's backward).
 */
int infini_attn_backward_ex(const void* q, const void* k, const void* v, const float* beta,
                            const float* M_in, const float* z_in, const void* dout,
                            const float* dM_out, const float* dz_out, void* dq, void* dk,
                            void* dv, float* dbeta, float* dM_in, float* dz_in, int B, int H,
                            long long L, int N, int d, int mode, const infini_attn_opts_t* opts,
                            void* stream);

/* Scratch bytes infini_attn_backward needs for these sizes (0 when the sizes are
 * not supported or L = 0). */
size_t infini_attn_backward_workspace_size(int B, int H, long long L, int N, int d, int mode);

/*
 * Device-side status of earlier calls on the current device: INFINI_OK, or
 * INFINI_ERR_TIMEOUT when a bounded wait inside a kernel ran out (the kernel
 * then stopped early and its outputs are invalid). Synchronises the device,
 * then clears the flag.
 */
int infini_attn_device_status(void);

/*
 * Runs one kernel whose only work is a bounded wait, on a barrier that nothing
 * arrives at, for about timeout_ns nanoseconds; it exists to exercise the
 * timeout path above (expected result: INFINI_ERR_TIMEOUT from
 * infini_attn_device_status afterwards).
 */
int infini_attn_selftest_timeout(long long timeout_ns, void* stream);

/* Text for a status code (static storage). */
const char* infini_attn_strerror(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int infini_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* INFINI_ATTN_H */
