/*
 * gdn.h -- C ABI of libgdn.so: the gated delta rule (Gated DeltaNet core) on
 * NVIDIA B200 (sm_100a).
 *
 * The operation is the gated delta rule as defined by the "手撕Qwen3-Next"
 * walkthrough (wkq9411.github.io, Code-Qwen3-Next), section 一(一)5
 * "应用 Gated Delta Rule": per v-head, with state S in R^{Dk x Dv},
 *
 *     q_hat = q / sqrt(sum q^2 + 1e-6) * scale,   k_hat = k / sqrt(sum k^2 + 1e-6)
 *     S <- S * exp(g_t)
 *     delta = beta_t (v_t - S^T k_hat)            (S^T k_hat: the value k_hat retrieves)
 *     S <- S + k_hat delta^T
 *     o_t = S^T q_hat                              (after token t's own write)
 *
 * gdn_chunk_fwd computes it for whole sequences with the chunkwise algorithm of
 * section 5(1) (prefill); gdn_recurrent_step advances every sequence by one
 * token (decode, section 5(2)).  The L2 norm with eps inside the root follows
 * the PyPTO-Gym "Qwen3Next 样例" README (数学公式); the packed [T, N, D] layout
 * with cumulative sequence lengths follows its 参数说明 (act_seq_len).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE memory owned by the caller, contiguous,
 *     row-major, 16-byte aligned.  The library never allocates or frees.
 *   - Calls are asynchronous on `cuda_stream` (a cudaStream_t; NULL = legacy
 *     default stream) of the CURRENT device.
 *   - The return value is GDN_OK or a negative gdn_status_t.  Arguments are
 *     validated on the host before anything is launched; a rejected call
 *     launches nothing and writes nothing.
 *   - Numbers: g, beta and the states are fp32; q, k, v and out have the
 *     dtype `io_dtype`.  Every accumulation is fp32.
 *   - GQA: v-head h reads qk-head h / (Nv / Nqk)  (repeat_interleave of the
 *     walkthrough, section 4).
 */
#ifndef GDN_H_
#define GDN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_NULL = -1,           /* a required pointer is NULL */
    GDN_ERR_SHAPE = -2,          /* unsupported head count, head dim, chunk size or length */
    GDN_ERR_ALIGN = -3,          /* a tensor pointer is not 16-byte aligned */
    GDN_ERR_ALIAS = -4,          /* `out` overlaps an input, or `state` overlaps q/k/v/out */
    GDN_ERR_CUDA = -5,           /* a CUDA runtime call or kernel launch failed */
    GDN_ERR_DEVICE = -6,         /* the current device is not a compute capability 10.0 GPU */
    GDN_ERR_DEVICE_TIMEOUT = -7, /* a bounded in-kernel wait expired (see gdn_device_status) */
    GDN_ERR_SEQLENS = -8,        /* cu_seqlens contents inconsistent (see gdn_device_status) */
    GDN_ERR_GATE = -9            /* g > 0 or NaN reached the tensor-core kernel (see gdn_device_status) */
} gdn_status_t;

typedef enum { GDN_DTYPE_F32 = 0, GDN_DTYPE_BF16 = 1 } gdn_dtype_t;

/* Kernel family for gdn_chunk_fwd.  AUTO picks the tensor-core kernel where it
 * applies (bf16 io, Dk = Dv = 128, chunk_size 64) and the SIMT kernel
 * otherwise: fp32 io, Dk or Dv = 64, or chunk_size 128.  The SIMT kernel keeps
 * fp32 accuracy (fp32 FMAs, and warp-level TF32 MMAs with each operand split
 * into two TF32 parts) and is several times slower per token; since the result
 * does not depend on chunk_size beyond rounding, bf16 callers get the fast path
 * with chunk_size 64. */
typedef enum { GDN_KERNEL_AUTO = 0, GDN_KERNEL_SIMT = 1, GDN_KERNEL_TC = 2 } gdn_kernel_t;

/* Shapes and options shared by both calls. */
typedef struct {
    int32_t num_qk_heads;  /* Nqk >= 1 */
    int32_t num_v_heads;   /* Nv >= 1, Nv % Nqk == 0 */
    int32_t head_k_dim;    /* Dk in {64, 128} */
    int32_t head_v_dim;    /* Dv in {64, 128} */
    int32_t io_dtype;      /* gdn_dtype_t of q, k, v, out */
    int32_t qk_l2norm;     /* 1: L2-normalise q and k in-kernel (eps 1e-6); 0: use as given */
    float scale;           /* query scale; <= 0 selects 1/sqrt(Dk) */
    int32_t kernel;        /* gdn_kernel_t; 0 = automatic */
} gdn_params_t;

/*
 * gdn_chunk_fwd -- chunked prefill over a packed batch of N sequences.
 *
 * Walkthrough section 5(1) steps a-g (torch_chunk_gated_delta_rule), per
 * sequence; the PyPTO README's fused chunk_gated_delta_rule interface.
 *
 *   q, k           [T, Nqk, Dk]  io_dtype
 *   v              [T, Nv, Dv]   io_dtype
 *   g, beta        [T, Nv]       fp32   (g = log of the decay, beta = write strength).
 *                  g <= 0 (a decay, as the layer's gate always is) where the
 *                  tensor-core kernel runs: it splits the in-chunk decay into
 *                  factors that are at most 1.  That kernel checks every gate
 *                  it loads; a g > 0 or NaN leaves its results undefined and is
 *                  reported by gdn_device_status as GDN_ERR_GATE.  The CUDA-core
 *                  kernel (GDN_KERNEL_SIMT) takes any finite g.
 *   initial_state  [N, Nv, Dk, Dv] fp32 (Dk rows, Dv contiguous) or NULL for zeros
 *   cu_seqlens     [N + 1] int32 device array: cu[0] = 0, non-decreasing, cu[N] = T;
 *                  sequence n owns tokens [cu[n], cu[n+1]) and starts from
 *                  initial_state[n].  NULL means N equal sequences of T / N
 *                  tokens (T % N must be 0).  The contents are checked on the
 *                  device: every kernel clamps each sequence's bounds to
 *                  0 <= cu[n] <= cu[n+1] <= T, so nothing is read or written
 *                  outside the tensors, and a violation (out of order, out of
 *                  range, cu[0] != 0 or cu[N] != T) is reported by
 *                  gdn_device_status as GDN_ERR_SEQLENS; the results of the
 *                  sequences involved are then undefined.
 *   num_seqs       N >= 1 (N <= 65535)
 *   total_tokens   T >= 0 (T < 2^31)
 *   chunk_size     C in {64, 128}: the chunk length of the chunkwise algorithm.
 *                  Every sequence has its own chunk grid starting at cu[n]; its
 *                  tail chunk is processed as if zero padded.  The result does
 *                  not depend on C beyond rounding.
 *   out            [T, Nv, Dv] io_dtype; must not overlap any input
 *   final_state    [N, Nv, Dk, Dv] fp32 or NULL; may be the same buffer as
 *                  initial_state (updated in place); other overlaps are rejected
 *   p              shapes and options (see gdn_params_t)
 *
 * Zero-length sequences are allowed: their final_state equals their initial state.
 * With total_tokens = 0 the token tensors (q, k, v, g, beta, out) are not read or
 * written and may be NULL; final_state then receives initial_state (or zeros).
 */
int gdn_chunk_fwd(const void *q, const void *k, const void *v,
                  const float *g, const float *beta,
                  const float *initial_state,
                  const int32_t *cu_seqlens,
                  int32_t num_seqs, int64_t total_tokens, int32_t chunk_size,
                  void *out, float *final_state,
                  const gdn_params_t *p, void *cuda_stream);

/*
 * gdn_recurrent_step -- one decode token for each of N sequences.
 *
 * Walkthrough section 5(2) (torch_recurrent_gated_delta_rule) with one token.
 * Equal to gdn_chunk_fwd on T = N sequences of length 1 with
 * final_state = initial_state = state.
 *
 *   q, k     [N, Nqk, Dk]   io_dtype
 *   v        [N, Nv, Dv]    io_dtype
 *   g, beta  [N, Nv]        fp32
 *   state    [N, Nv, Dk, Dv] fp32, read and updated IN PLACE
 *   out      [N, Nv, Dv]    io_dtype; must not overlap any input or the state
 *   num_seqs N >= 1
 */
int gdn_recurrent_step(const void *q, const void *k, const void *v,
                       const float *g, const float *beta,
                       float *state, void *out, int32_t num_seqs,
                       const gdn_params_t *p, void *cuda_stream);

/*
 * gdn_chunk_fwd_slots / gdn_recurrent_step_slots -- the same two calls with the
 * recurrent states kept in a pool of rows, as a serving cache holds them (the
 * walkthrough's Cache section: one [Nv, Dk, Dv] recurrent state per sequence),
 * addressed through per-sequence slot ids and updated in place:
 *
 *   state_pool  [num_slots, Nv, Dk, Dv] fp32: row slot_ids[n] is the state of
 *               sequence n on entry and is overwritten with its state on exit
 *   slot_ids    [N] int32 device array, 4-byte aligned.  An id outside
 *               [0, num_slots) marks a padding sequence: it is processed from a
 *               zero state and nothing is stored for it (gdn_recurrent_step_slots
 *               writes zeros to its output row).  Active sequences must have
 *               distinct ids; contents are not otherwise validated.
 *   num_slots   >= 1
 *
 * gdn_chunk_fwd_slots with cu_seqlens advances every sequence by its own number
 * of tokens (1 for a plain decode step, more for a multi-token step or a
 * prefill into the cache); it always uses the chunked kernels.  The pool and
 * the slot ids count as inputs for the overlap rules; the pool may not
 * overlap out.  Other arguments and status codes are those of gdn_chunk_fwd /
 * gdn_recurrent_step.
 */
int gdn_chunk_fwd_slots(const void *q, const void *k, const void *v,
                        const float *g, const float *beta,
                        float *state_pool, const int32_t *slot_ids, int32_t num_slots,
                        const int32_t *cu_seqlens,
                        int32_t num_seqs, int64_t total_tokens, int32_t chunk_size,
                        void *out, const gdn_params_t *p, void *cuda_stream);

int gdn_recurrent_step_slots(const void *q, const void *k, const void *v,
                             const float *g, const float *beta,
                             float *state_pool, const int32_t *slot_ids, int32_t num_slots,
                             void *out, int32_t num_seqs,
                             const gdn_params_t *p, void *cuda_stream);

/*
 * gdn_chunk_fwd_gated / gdn_recurrent_step_gated -- the same two calls with the
 * gate formed in-kernel from the layer's raw projections, as in the walkthrough's
 * section 一(一)4 (形状调整):
 *
 *   beta = sigmoid(b),   g = -exp(A_log[h]) * softplus(a + dt_bias[h]),
 *   softplus(x) = log(1 + exp(x))   (evaluated as max(x,0) + log1p(exp(-|x|)))
 *
 *   a, b      [T, Nv] (prefill) or [N, Nv] (decode), fp32: take the places of g, beta
 *   A_log     [Nv] fp32, the log of the per-head decay rate A > 0
 *   dt_bias   [Nv] fp32
 *
 * A_log and dt_bias must be non-NULL and 4-byte aligned; every other argument,
 * shape rule, overlap rule and status code is that of gdn_chunk_fwd /
 * gdn_recurrent_step (a, b, A_log, dt_bias count as inputs).  The gate is
 * evaluated in fp32 with the accurate CUDA expf / log1pf.
 */
int gdn_chunk_fwd_gated(const void *q, const void *k, const void *v,
                        const float *a, const float *b,
                        const float *A_log, const float *dt_bias,
                        const float *initial_state,
                        const int32_t *cu_seqlens,
                        int32_t num_seqs, int64_t total_tokens, int32_t chunk_size,
                        void *out, float *final_state,
                        const gdn_params_t *p, void *cuda_stream);

int gdn_recurrent_step_gated(const void *q, const void *k, const void *v,
                             const float *a, const float *b,
                             const float *A_log, const float *dt_bias,
                             float *state, void *out, int32_t num_seqs,
                             const gdn_params_t *p, void *cuda_stream);

/*
 * gdn_ext_t -- optional fusions around the core, taken by gdn_chunk_fwd_ex and
 * gdn_recurrent_step_ex.  A NULL pointer or an all-zero struct selects none,
 * and the _ex calls then equal gdn_chunk_fwd / gdn_recurrent_step.  Fields:
 *
 *   A_log, dt_bias   fused gate, as the _gated calls: both non-NULL => the g and
 *                    beta arguments hold the raw projections a and b.
 *   slot_ids,        slot pool, as the _slots calls: non-NULL slot_ids => the
 *   num_slots        state arguments address a pool [num_slots, Nv, Dk, Dv];
 *                    gdn_chunk_fwd_ex then requires final_state == initial_state
 *                    (the pool, non-NULL).
 *   norm_z,          gated RMSNorm epilogue (RMSNormGated of the walkthrough's
 *   norm_weight,     sections 一(一)1 and 6): non-NULL norm_z => every (token,
 *   norm_eps         v-head) row o of Dv outputs is stored as
 *                        y = o / sqrt(mean(o^2) + norm_eps) * norm_weight * silu(z),
 *                        silu(x) = x / (1 + exp(-x)),
 *                    computed in fp32 (where gdn_chunk_fwd_ex's pass stores bf16,
 *                    silu is evaluated as h + h tanh(h), h = x / 2, with the
 *                    hardware tanh approximation: error at most |x| 2^-12).  gdn_recurrent_step_ex normalises the fp32 o
 *                    before its one rounding to io_dtype; gdn_chunk_fwd_ex stores o
 *                    and then rewrites each row in place (gdn_gated_rmsnorm), so
 *                    there o is rounded to io_dtype once before the norm.
 *                    norm_z has the shape and dtype of `out` ([T or N, Nv, Dv]),
 *                    norm_weight is [Dv] fp32, both 16-byte aligned and counted as
 *                    inputs for the overlap rules; norm_eps is finite and >= 0
 *                    (the layer's default is 1e-6).  A padding slot's decode row
 *                    stays zero.
 *   conv_x,          causal conv fused ahead of the decode step (gdn_recurrent_step_ex
 *   conv_state,      only): non-NULL conv_x => q, k, v must be NULL and the step
 *   conv_weight,     forms them in-kernel from the packed projection, exactly as
 *   conv_bias,       gdn_qkv_conv_update would (without rounding them to io_dtype):
 *   conv_kernel_size   conv_x      [N, C] io_dtype, C = 2 Nqk Dk + Nv Dv, 16-byte aligned
 *                      conv_state  [N, C, K] io_dtype (rows as the recurrent state:
 *                                  with slot_ids, [num_slots, C, K] and the same
 *                                  slots), 16-byte aligned, updated in place
 *                      conv_weight [C, K] fp32;  conv_bias [C] fp32 or NULL
 *                      conv_kernel_size K in [1, 4]
 *                    The Nv / Nqk v-heads of a qk-head run as one thread-block
 *                    cluster, so Nv / Nqk must be at most 8 (else GDN_ERR_SHAPE).
 *                    The fusion saves a launch, not time: on B200, for 256
 *                    sequences x 32 v-heads (D = 128), it measured about 207 us
 *                    per step against about 183 us for gdn_qkv_conv_update
 *                    followed by gdn_recurrent_step, because the CTAs of a
 *                    cluster must be co-scheduled.  Where time matters, use the
 *                    two calls.
 */
typedef struct {
    const float *A_log;
    const float *dt_bias;
    const int32_t *slot_ids;
    int32_t num_slots;
    const void *norm_z;
    const float *norm_weight;
    float norm_eps;
    const void *conv_x;
    void *conv_state;
    const float *conv_weight;
    const float *conv_bias;
    int32_t conv_kernel_size;
} gdn_ext_t;

/*
 * gdn_chunk_fwd_ex / gdn_recurrent_step_ex -- gdn_chunk_fwd / gdn_recurrent_step
 * with the fusions selected in `ext` (any combination).  Every argument, shape
 * rule, overlap rule and status code of the plain calls applies; `ext` adds its
 * own (GDN_ERR_NULL for a half-given gate, a norm_z without norm_weight or a
 * conv_x without conv_state / conv_weight; GDN_ERR_SHAPE for num_slots < 1, a
 * bad norm_eps or conv_kernel_size, q / k / v given together with conv_x, or
 * conv_x on gdn_chunk_fwd_ex, whose prefill conv is gdn_qkv_conv_fwd;
 * GDN_ERR_ALIGN; GDN_ERR_ALIAS when an output overlaps any of these inputs).
 */
int gdn_chunk_fwd_ex(const void *q, const void *k, const void *v,
                     const float *g, const float *beta,
                     const float *initial_state,
                     const int32_t *cu_seqlens,
                     int32_t num_seqs, int64_t total_tokens, int32_t chunk_size,
                     void *out, float *final_state,
                     const gdn_params_t *p, const gdn_ext_t *ext, void *cuda_stream);

int gdn_recurrent_step_ex(const void *q, const void *k, const void *v,
                          const float *g, const float *beta,
                          float *state, void *out, int32_t num_seqs,
                          const gdn_params_t *p, const gdn_ext_t *ext, void *cuda_stream);

/*
 * gdn_gated_rmsnorm -- the gated RMSNorm epilogue on its own (RMSNormGated,
 * walkthrough sections 一(一)1 and 6), for rows produced elsewhere:
 *
 *   y[r, :] = o[r, :] / sqrt(mean(o[r, :]^2) + eps) * weight * silu(z[r, :])
 *
 *   o, z, y   [rows, dim] io_dtype (gdn_dtype_t), 16-byte aligned; y may be o
 *             (in place) but must not overlap z or weight otherwise
 *   weight    [dim] fp32, 16-byte aligned
 *   rows      >= 0 (< 2^31);  dim in {64, 128};  eps finite, >= 0.  With rows == 0
 *             the call does nothing and returns GDN_OK (the pointers may be NULL).
 * Arithmetic is fp32; for bf16 io silu is evaluated as h + h tanh(h), h = x / 2,
 * with the hardware tanh approximation (error at most |x| 2^-12).
 */
int gdn_gated_rmsnorm(const void *o, const void *z, const float *weight, float eps,
                      void *y, int64_t rows, int32_t dim, int32_t io_dtype,
                      void *cuda_stream);

/*
 * gdn_qkv_conv_fwd / gdn_qkv_conv_update -- the causal depthwise conv1d + SiLU
 * that turns the layer's packed projection mixed_qkv = [q | k | v] into the
 * q, k, v of the calls above (walkthrough section 一(一)3, qkv 卷积部分; the
 * decode form is its torch_causal_conv1d_update).  With C = 2 Nqk Dk + Nv Dv
 * channels (shapes and io_dtype from p; p's qk_l2norm, scale and kernel are not
 * used) and K = kernel_size taps:
 *
 *   y[t, c] = silu(bias[c] + sum_{i < K} weight[c, i] * in(t - (K - 1) + i))
 *
 * where in(p) is the sequence's input at position p, or for p < 0 the window
 * cached before it, conv_state[n, c, K + p] (zeros when no state is given).
 * Channel c < Nqk Dk is stored to q[t, c], c < 2 Nqk Dk to k[t, c - Nqk Dk], the
 * rest to v[t, c - 2 Nqk Dk]; q, k are [rows, Nqk, Dk] and v [rows, Nv, Dv] in
 * io_dtype, as gdn_chunk_fwd / gdn_recurrent_step read them.  A conv_state row
 * is [C, K] in io_dtype holding the last K inputs (pre-convolution), the
 * newest at index K - 1.  All arithmetic is fp32; silu(x) = x / (1 + exp(-x)),
 * for bf16 io evaluated as h + h tanh(h), h = x / 2, with the hardware tanh
 * approximation (error at most |x| 2^-12, under the rounding of a bf16 output
 * for x > 0).
 *
 *   mixed_qkv   [T, C] (prefill, packed sequences) or [N, C] (decode), io_dtype
 *   weight      [C, K] fp32, 16-byte aligned (read as 16-byte vectors);
 *               bias [C] fp32 or NULL, 4-byte aligned
 *   kernel_size K in [1, 4]
 *
 * gdn_qkv_conv_fwd (prefill over N sequences, cu_seqlens as in gdn_chunk_fwd):
 *   total_tokens    T >= 0; with T = 0, mixed_qkv, q, k and v may be NULL
 *   conv_state_in   [N, C, K] or NULL (each sequence starts after zeros)
 *   conv_state_out  [N, C, K] or NULL: the last K inputs of [window, sequence]
 *                   (zero filled on the left when fewer exist); may be
 *                   conv_state_in (updated in place), may not overlap it otherwise
 * gdn_qkv_conv_update (one token per sequence):
 *   conv_state      [N, C, K] (or [num_slots, C, K] with slot_ids), updated in
 *                   place: shifted by one, the new input at index K - 1
 *   slot_ids        [N] int32 or NULL, as gdn_recurrent_step_slots: an id
 *                   outside [0, num_slots) is a padding sequence (zero q, k, v;
 *                   no state touched)
 *
 * q, k, v and the output state may not overlap the inputs or each other.
 * Status codes as for gdn_chunk_fwd.
 */
int gdn_qkv_conv_fwd(const void *mixed_qkv, const float *weight, const float *bias,
                     const void *conv_state_in, const int32_t *cu_seqlens,
                     int32_t num_seqs, int64_t total_tokens, int32_t kernel_size,
                     void *q, void *k, void *v, void *conv_state_out,
                     const gdn_params_t *p, void *cuda_stream);

int gdn_qkv_conv_update(const void *mixed_qkv, const float *weight, const float *bias,
                        void *conv_state, const int32_t *slot_ids, int32_t num_slots,
                        int32_t num_seqs, int32_t kernel_size,
                        void *q, void *k, void *v,
                        const gdn_params_t *p, void *cuda_stream);

/*
 * gdn_device_status -- read and clear, in one atomic step ordered on
 * `cuda_stream`, the library's device-side status word for the current
 * device, then synchronise the stream.  Every kernel of the library reports
 * into that word, whatever stream it ran on.  Returns, for what was reported
 * since the last call (in this order of precedence):
 *   GDN_ERR_DEVICE_TIMEOUT  a kernel gave up a bounded wait (its outputs are undefined)
 *   GDN_ERR_SEQLENS         a kernel met an inconsistent cu_seqlens (see gdn_chunk_fwd)
 *   GDN_ERR_GATE            the tensor-core chunk kernel met a gate g > 0 or NaN
 *   GDN_OK                  nothing,
 * or GDN_ERR_CUDA if the stream reported an error.  Reports of kernels still
 * running on other streams count towards the next call.  Calls from several
 * host threads at once may swap their results.
 */
int gdn_device_status(void *cuda_stream);

/*
 * gdn_selftest_wait_timeout -- self-test of the device-side failure detection.
 * Launches one CTA on `cuda_stream` that waits, with the library's bounded
 * mbarrier wait, on a barrier nothing arrives on; after limit_us microseconds
 * (1 .. 2,000,000) the wait gives up and records the timeout in the status word
 * that gdn_device_status reads, and the CTA returns.  Nothing faults or hangs,
 * and the context stays usable.  Returns GDN_OK once launched.
 */
int gdn_selftest_wait_timeout(int64_t limit_us, void *cuda_stream);

/* Human-readable name of a status code (static storage; never NULL). */
const char *gdn_status_string(int status);

/* ABI version: (major << 16) | minor. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
