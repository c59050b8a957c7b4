/*
 * gdr.h -- C ABI of the B200 (sm_100a) gated delta rule library, libgdr.so.
 *
 * The gated delta rule keeps, per (batch row b, value head h), a state
 * S in R^{Dk x Dv} (row i over the key dimension, column j over the value
 * dimension, row-major) and for each token t applies, in this order:
 *
 *     S   <- S * exp(g_t)            (and, for decode, row i also * exp(gk_t[i]))
 *     m    = k_t^T S                 (readout, length Dv)
 *     d    = beta_t * (v_t - m)      (delta)
 *     S   <- S + k_t d^T             (rank-1 write)
 *     o_t  = (scale * q_t)^T S       (output)
 *
 * Sources: the torch_recurrent_gated_delta_rule token loop of the
 * transformers GatedDeltaNet layer (blog "gated-delta-net" page), delta_step
 * in inferencelayer deltanet.rs, and the algorithm statement of the
 * lite_boost recurrent_gated_delta_rule and chunk_gated_delta_rule operators.
 *
 * Conventions for every entry point:
 *   - Tensors are dense, row-major (C-contiguous), in DEVICE memory of the
 *     current CUDA device, in the BNSD layout of the lite_boost operators:
 *       q, k           (B, Nk, S, Dk)
 *       v, out         (B, Nv, S, Dv)
 *       beta, g        (B, Nv, S)
 *       gk             (B, Nv, S, Dk)
 *       initial/final  (B, Nv, Dk, Dv)
 *       state_pool     (slots, Nv, Dk, Dv)
 *   - Grouped heads: Nv must be a multiple of Nk; value head h reads key head
 *     h / (Nv / Nk) (contiguous groups, the repeat_interleave grouping).
 *   - dtype names the type of q, k, v, beta, the state and out: GDR_F32,
 *     GDR_BF16 or GDR_F16 (the chunk_gated_delta_rule operator lists fp16 and
 *     bf16 inputs).  g, gk and the prologue's a, A_log, dt_bias are always fp32.
 *     bf16 and fp16 prefill with Dk = Dv = 128 run on the tensor cores (fp32
 *     accumulation and state, MMA operand copies in the input type); other
 *     head sizes and fp32 run the CUDA-core kernel (fp32 arithmetic, one
 *     rounding of each output).  Decode takes a state of GDR_F32, GDR_BF16 or
 *     GDR_F16 (an fp16 state needs fp16 inputs, fp16 inputs an fp16 or fp32
 *     state; other pairs: GDR_ERR_DTYPE).
 *     Index arrays are int32.  Stores to bf16 round to nearest even, once.
 *   - The caller owns every buffer.  The library allocates no device memory
 *     and keeps no pointer after a call returns; the scratch of the
 *     tensor-core prefill's two-kernel schedule is an optional caller-owned
 *     workspace sized by gdr_chunk_fwd_workspace().
 *     Work is enqueued on
 *     `stream` (a cudaStream_t; NULL = the legacy default stream) and runs
 *     asynchronously: the call returns before the kernels finish.
 *   - Host-side argument checks run before anything is launched; on a non-zero
 *     status nothing is launched and no buffer is touched.
 *   - Device-side checks (slot index outside [0, slots), length outside
 *     [0, S]) never trap: the affected sequence is skipped, its output rows
 *     are written as zero, and a bit is set in the device error word read by
 *     gdr_get_error().
 *   - g and gk are not range-checked (the lite_boost operators document that a
 *     min/max reduction would cost visible time on the inference path);
 *     positive values give meaningless but finite-or-inf results.
 */
#ifndef GDR_H
#define GDR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *gdr_stream_t;

/* Status codes.  The Python binding maps GDR_ERR_SHAPE to ValueError (the
 * shape errors the lite_boost operators raise as ValueError) and every other
 * non-zero status to RuntimeError. */
typedef enum gdr_status {
    GDR_OK = 0,
    GDR_ERR_SHAPE = 1,       /* Nv % Nk != 0, sizes < 0, decode S > 8, slots < 1, ... */
    GDR_ERR_DTYPE = 2,       /* unknown dtype code or unsupported dtype combination */
    GDR_ERR_NULL = 3,        /* a required pointer is NULL */
    GDR_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned */
    GDR_ERR_UNSUPPORTED = 5, /* valid per the API but not built: Dk or Dv not in {16,32,64,128} */
    GDR_ERR_DEVICE = 6,      /* no usable device, or it is not sm_100 */
    GDR_ERR_LAUNCH = 7,      /* a kernel launch or a CUDA call failed */
    GDR_ERR_WORKSPACE = 8    /* ws_bytes is smaller than gdr_chunk_fwd_workspace() returns */
} gdr_status;

typedef enum gdr_dtype { GDR_F32 = 0, GDR_BF16 = 1, GDR_F16 = 2 } gdr_dtype;

/* Bits of the device error word (gdr_get_error). */
#define GDR_DEVERR_SLOT_INDEX 0x1u /* a referenced slot index was outside [0, slots) */
#define GDR_DEVERR_LENGTH 0x2u     /* a length was outside [0, S] */
#define GDR_DEVERR_TIMEOUT 0x4u    /* a kernel's bounded wait for its own copies or for another of its warp
                                      groups ran out: it released what it held and returned early, so the
                                      call's outputs are incomplete (not expected in normal operation) */

/*
 * Optional fused prologue (the layer's pre-processing, computed in fp32
 * inside the kernels' load stage so it costs no extra pass over memory).
 * Source: the transformers GatedDeltaNet forward (blog page: beta =
 * b.sigmoid(), g = -A_log.exp() * softplus(a + dt_bias), l2norm of q and k
 * with eps 1e-6) and deltanet.rs (l2norm with eps INSIDE the square root).
 */
typedef struct gdr_prologue {
    int l2norm_qk;         /* non-zero: q and k are raw; each row x becomes x / sqrt(sum x^2 + eps) */
    float eps;             /* the l2norm epsilon (1e-6 in the layer) */
    int beta_logits;       /* non-zero: the beta buffer holds logits b and beta = 1 / (1 + exp(-b)) */
    const float *A_log;    /* non-NULL: the g buffer holds the raw a (fp32) and
                              g = -exp(A_log[h]) * softplus(a + dt_bias[h]); device, (Nv) */
    const float *dt_bias;  /* device, (Nv); required when A_log is non-NULL */
} gdr_prologue;

/*
 * Optional output epilogue: the gated RMSNorm the layer applies to each head's
 * output row before its output projection, fused into the call.  Source: the
 * per-head gated RMSNorm of deltanet.rs and of its WGSL core shader (mean of
 * the squares over the head's Dv outputs, eps inside the square root, times the
 * norm weight and silu of the head's slice of z), applied by the transformers
 * layer as self.norm(core_attn_out, z) (blog "gated-delta-net" page; its
 * comment names the gate sigmoid(z), both code listings use silu).
 *
 *   z        device (B, Nv, S, Dv) in dtype: the layer's output gate branch
 *   norm_w   device fp32 (Dv): the RMSNorm weight, shared by all heads
 *   eps      added to the mean square inside the square root (>= 0)
 *
 * With it, out row (b, h, t) for t < L_b holds, computed in fp32 and rounded
 * once to dtype:
 *     o / sqrt(mean_j o_j^2 + eps) * norm_w * silu(z),  silu(x) = x / (1 + e^{-x})
 * where o is the row the rule produces; padding rows stay zero.  The
 * tensor-core prefill (bf16 or fp16, Dk = Dv = 128) applies it to the fp32 row
 * before rounding; the other paths apply it to the row already stored in
 * dtype (for a 16-bit dtype that rounds o once more, within its tolerance).  z and norm_w must be 16-byte aligned.
 */
typedef struct gdr_epilogue {
    const void *z;
    const float *norm_w;
    float eps;
} gdr_epilogue;

/*
 * Bytes of device workspace the fastest schedule of a gdr_chunk_fwd call with
 * these sizes wants (0 if it wants none).  The tensor-core path (bf16 or fp16,
 * Dk = Dv = 128) has two schedules:
 *   - one kernel, one CTA per (b, value head) chain, each chain solving its
 *     chunks' WY systems itself; needs no workspace;
 *   - two kernels: the WY transform of every 64-token chunk solved at once on
 *     every SM, keeping per (b, value head, chunk) the 64 x 64 matrix
 *     (I + A)^{-1} diag(beta) in the input dtype and six vectors of 64 floats
 *     (the chunk's gate and norm factors), then the chains.  Workspace:
 *     B * Nv * ceil(S / 64) * (8192 + 1536) bytes.
 * The two-kernel schedule is asked for when the chains fill at most a third of
 * the current device's SMs (B * Nv * 3 <= SMs; a device that cannot be asked
 * counts as 148), where the one-kernel schedule would leave most SMs idle.
 * Other shapes, fp32 and invalid sizes give 0 (the call itself reports the
 * latter).  Source: the lite_boost chunk_gated_delta_rule operator
 * (caller-owned buffers) and the order of torch_chunk_gated_delta_rule, which
 * forms every chunk's attn/T solve before the inter-chunk loop.
 */
size_t gdr_chunk_fwd_workspace(int B, int Nk, int Nv, int S, int Dk, int Dv, gdr_dtype dtype);

/*
 * Chunked prefill.  Source: lite_boost chunk_gated_delta_rule (arguments,
 * BNSD layout, GQA, variable lengths with padding written as zero, optional
 * gate, final state) and torch_chunk_gated_delta_rule (chunk size 64,
 * cumulative gate, WY/UT transform, inter-chunk carry).
 *
 *   q, k, v, beta          device, see layouts above (raw q, k and logits when
 *                          the prologue asks for them)
 *   g                      device fp32 (B, Nv, S) log-decay, or NULL: no decay
 *                          (with prologue->A_log set: the raw a, required)
 *   initial_state          device (B, Nv, Dk, Dv) or NULL: zeros
 *   actual_seq_lengths     device int32 (B) or NULL: every sequence has S
 *                          tokens.  Tokens t >= L_b are padding: their input
 *                          contents are ignored (they may hold any finite or
 *                          non-finite values) and out rows t >= L_b are zero.
 *                          L_b = 0 gives final_state = initial_state exactly.
 *   scale                  multiplies q before the rule (1/sqrt(Dk) in the layer)
 *   epilogue               NULL, or the fused gated RMSNorm of the out rows
 *                          (see gdr_epilogue)
 *   out                    device (B, Nv, S, Dv), written in full
 *   final_state            device (B, Nv, Dk, Dv) or NULL: not written.  It
 *                          may alias initial_state (in-place update).
 *   workspace, ws_bytes    NULL and 0, or device scratch of at least
 *                          gdr_chunk_fwd_workspace(B, Nk, Nv, S, Dk, Dv, dtype)
 *                          bytes, owned by the caller, 16-byte aligned.  With
 *                          it, the schedule the query sized runs; without it
 *                          (or when the query gives 0) the one-kernel
 *                          schedule.  Both give the same result up to rounding.
 *                          Its contents on entry do not matter and on return
 *                          are unspecified; two calls in flight at once need
 *                          separate workspaces.
 * Constraints: B, S >= 0; Nk, Nv >= 1; Nv % Nk == 0; Dk, Dv in {16,32,64,128};
 * every pointer 16-byte aligned.  An epilogue with a NULL z or norm_w returns
 * GDR_ERR_NULL, one with eps < 0 (or NaN) GDR_ERR_SHAPE.  A workspace shorter
 * than the query returns GDR_ERR_WORKSPACE.  bf16 or fp16 with
 * Dk = Dv = 128 runs on the tensor-core (tcgen05) path in one of the two
 * schedules above; other shapes and fp32 run the CUDA-core path.  Without g
 * (NULL, the operator's hasGamma = 0) a build without the gate arithmetic
 * runs.
 */
int gdr_chunk_fwd(const void *q, const void *k, const void *v, const void *beta, const float *g,
                  const void *initial_state, const int32_t *actual_seq_lengths, float scale, int B, int Nk,
                  int Nv, int S, int Dk, int Dv, gdr_dtype dtype, const gdr_prologue *prologue,
                  const gdr_epilogue *epilogue, void *out, void *final_state, void *workspace, size_t ws_bytes,
                  gdr_stream_t stream);

/*
 * The chunked prefill for callers that cannot allocate device memory: code in
 * a framework hook or plug-in that only receives one operation's tensors, a
 * serving loop whose memory is all reserved by its own pool, a runtime with no
 * allocator to call on this path.  It takes the arguments of gdr_chunk_fwd
 * without workspace and ws_bytes, and computes the same result; the scratch
 * the tensor-core path needs is instead a fixed 16 MiB array compiled into the
 * library (one per GPU that loads the library, held until the process exits).
 * No passage of the operator pages corresponds to this entry point: it exists
 * for the memory discipline of such callers.
 *   - It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - Sizes whose workspace (gdr_chunk_fwd_workspace) exceeds 16 MiB, that is
 *     the two-kernel schedule with B * Nv * ceil(S / 64) > 1724, return
 *     GDR_ERR_WORKSPACE without launching anything.  Sizes whose query is 0
 *     (the one-kernel schedule, the CUDA-core path) need no scratch and have
 *     no such limit.
 *   - Every call shares the one array per device, so two calls that overlap on
 *     the GPU (on different streams, or from different host threads, without
 *     ordering between them) race and give wrong results.  Calls ordered on one
 *     stream are fine; the array keeps the last call's contents, which no later
 *     call depends on.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 * Other arguments, checks, layouts and errors are those of gdr_chunk_fwd.
 */
int gdr_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *beta, const float *g,
                          const void *initial_state, const int32_t *actual_seq_lengths, float scale, int B, int Nk,
                          int Nv, int S, int Dk, int Dv, gdr_dtype dtype, const gdr_prologue *prologue,
                          const gdr_epilogue *epilogue, void *out, void *final_state, gdr_stream_t stream);

/*
 * Recurrent decode over a pool of state slots.  Source: lite_boost
 * recurrent_gated_delta_rule (state pool, ssm_state_indices with one slot per
 * flattened token, gk, num_accepted_tokens, S <= 8, the decay
 * S * exp(g) * exp(gk)).
 *
 *   q, k, v, beta, g       as for gdr_chunk_fwd (g may be NULL: no decay)
 *   gk                     device fp32 (B, Nv, S, Dk) per-key-row log-decay,
 *                          or NULL
 *   state_pool             device (slots, Nv, Dk, Dv) in state_dtype, read and
 *                          updated IN PLACE.  Slots no token commits to are
 *                          left byte-identical.
 *   ssm_state_indices      device int32 (B * S): slot of token (b, t) is
 *                          ssm_state_indices[b * S + t]
 *   actual_seq_lengths     device int32 (B): tokens processed for sequence b,
 *                          in [0, S]; out rows t >= L_b are zero
 *   num_accepted_tokens    device int32 (B), or NULL (= actual_seq_lengths)
 *   epilogue               NULL, or the gated RMSNorm of the out rows (see
 *                          gdr_epilogue)
 *   out                    device (B, Nv, S, Dv), written in full
 * Reading of num_accepted_tokens (the operator defines it only as the count of
 * accepted tokens, equal to the lengths in plain inference): the chain starts
 * from slot ssm_state_indices[b * S]; all L_b tokens are processed and
 * output; the state after token t is committed to slot
 * ssm_state_indices[b * S + t] only when t < min(A_b, L_b).  Two sequences
 * must not reference the same slot (their updates would race).
 * Constraints: 1 <= S <= 8 (the operator is decode-only), slots >= 1, other
 * constraints as for gdr_chunk_fwd.  state_dtype may be GDR_F32 or GDR_BF16
 * with GDR_F32 or GDR_BF16 inputs; fp16 inputs take GDR_F16 or GDR_F32.
 */
int gdr_recurrent_step(const void *q, const void *k, const void *v, const void *beta, const float *g,
                       const float *gk, void *state_pool, int slots, const int32_t *ssm_state_indices,
                       const int32_t *actual_seq_lengths, const int32_t *num_accepted_tokens, float scale, int B,
                       int Nk, int Nv, int S, int Dk, int Dv, gdr_dtype dtype, gdr_dtype state_dtype,
                       const gdr_prologue *prologue, const gdr_epilogue *epilogue, void *out,
                       gdr_stream_t stream);

/*
 * The decode call with the speculative-decoding reading of num_accepted_tokens:
 * per-token state slots.  Source: the recurrent_gated_delta_rule operator
 * (lite_boost) gives num_accepted_tokens only as the number of accepted
 * tokens; in speculative decoding the previous step wrote the state after each
 * of its tokens to that token's own slot and A_b of them were accepted.  So
 * here the chain of sequence b starts from pool[ssm_state_indices[b*S + A_b - 1]]
 * and the state after every processed token t < L_b is written to
 * pool[ssm_state_indices[b*S + t]].  A_b must lie in [1, S] for a sequence with
 * L_b > 0 (otherwise the sequence is skipped, its out rows are zero and
 * GDR_DEVERR_LENGTH is set); num_accepted_tokens == NULL means A_b = 1.
 * Arguments, layouts and the other errors are those of gdr_recurrent_step.
 */
int gdr_recurrent_step_spec(const void *q, const void *k, const void *v, const void *beta, const float *g,
                            const float *gk, void *state_pool, int slots, const int32_t *ssm_state_indices,
                            const int32_t *actual_seq_lengths, const int32_t *num_accepted_tokens, float scale,
                            int B, int Nk, int Nv, int S, int Dk, int Dv, gdr_dtype dtype, gdr_dtype state_dtype,
                            const gdr_prologue *prologue, const gdr_epilogue *epilogue, void *out,
                            gdr_stream_t stream);

/*
 * Depthwise causal conv1d + SiLU over the fused q/k/v channels, with its state:
 * the step before the rule, writing the rule's q, k and v.  Source: the layer's
 * conv over mixed_qkv = cat(q, k, v) with causal_conv1d_fn (prefill) and
 * causal_conv1d_update (decode), conv_state = F.pad(mixed_qkv, (K - L, 0))
 * (blog "gated-delta-net" page), and the per-channel ring of the last K inputs
 * in deltanet.rs and its WGSL twin (shift, append, dot with the taps oldest
 * first, silu).
 *
 * For sequence b (L = L_b valid positions) and channel c:
 *     y[t, c] = silu(bias[c] + sum_{j<K} weight[c, j] * x[t - K + 1 + j, c]),  t < L
 * where the K positions before 0 come from conv_state_in (newest last; zeros
 * when it is NULL).  Computed in fp32, rounded once to dtype.
 *
 *   x                    device (B, S, C) channels last, C = 2*Nk*Dk + Nv*Dv: the
 *                        q channels (Nk heads of Dk), then k (Nk x Dk), then v (Nv x Dv)
 *   weight               device (C, K), taps oldest first
 *   bias                 device (C) or NULL: no bias
 *   conv_state_in        device (B, C, K) or NULL: zeros
 *   actual_seq_lengths   device int32 (B) or NULL: all S; positions t >= L_b are padding
 *   q, k, v              device outputs (B, Nk, S, Dk), (B, Nk, S, Dk), (B, Nv, S, Dv):
 *                        y split by channel and head; padding rows are zero
 *   conv_state_out       device (B, C, K) or NULL: the last K inputs of the history
 *                        (conv_state_in followed by x[0..L_b-1]); it may alias
 *                        conv_state_in (the in-place update of decode)
 * x, weight, bias, the states and the outputs are in dtype (GDR_F32,
 * GDR_BF16 or GDR_F16).  Constraints: B, S >= 0; Nk, Nv >= 1; Dk, Dv in {16,32,64,128};
 * 1 <= K <= 8 (4 in the layer); every pointer 16-byte aligned.  A length
 * outside [0, S] skips the sequence (outputs zero, state untouched) and sets
 * GDR_DEVERR_LENGTH.
 */
int gdr_conv1d(const void *x, const void *weight, const void *bias, const void *conv_state_in,
               const int32_t *actual_seq_lengths, int B, int S, int Nk, int Nv, int Dk, int Dv, int K,
               gdr_dtype dtype, void *q, void *k, void *v, void *conv_state_out, gdr_stream_t stream);

/*
 * Stand-alone prologue (the same arithmetic the fused prologue applies), for
 * callers that want the normalised tensors materialised.  Source: as for
 * gdr_prologue.
 *   q, k      device (B, Nk, S, Dk) raw, or NULL to skip; written to q_hat,
 *             k_hat (same dtype, may alias the inputs) as x / sqrt(sum x^2 + eps)
 *   b         device (B, Nv, S) logits in dtype, or NULL; beta = sigmoid(b)
 *             written to beta (dtype, may alias b)
 *   a         device fp32 (B, Nv, S), or NULL; g = -exp(A_log[h]) *
 *             softplus(a + dt_bias[h]) written to g (fp32, may alias a);
 *             A_log and dt_bias are device fp32 (Nv), required with a
 */
int gdr_prologue_apply(const void *q, const void *k, const void *b, const float *a, const float *A_log,
                       const float *dt_bias, float eps, int B, int Nk, int Nv, int S, int Dk, gdr_dtype dtype,
                       void *q_hat, void *k_hat, void *beta, float *g, gdr_stream_t stream);

/*
 * Returns in *device_error the device error word and clears it, in one atomic
 * step on `stream` (after the work already enqueued there), then waits for
 * the stream.  The word is one per device: it holds the GDR_DEVERR_* bits
 * raised by every kernel of this library on the current device since it was
 * last cleared, including kernels on other streams or from other host
 * threads, so a caller that needs per-call attribution serialises its calls.
 * Returns GDR_OK, or GDR_ERR_LAUNCH if a CUDA call failed (including an
 * earlier asynchronous kernel fault on the stream).
 */
int gdr_get_error(gdr_stream_t stream, int *device_error);

/*
 * Diagnostic hook for the bounded waits of the tensor-core prefill and of the
 * D = 128 decode kernel: their limit in nanoseconds for the calls that follow in
 * this process (0 restores the default of one second).  A limit shorter than a
 * kernel needs makes its waits run out: the kernel then drains its own copies
 * (and MMAs), returns early and sets GDR_DEVERR_TIMEOUT (outputs and, for
 * decode, the state pool incomplete).  Used by the tests of those paths; not
 * for production use.  Always returns GDR_OK.
 */
int gdr_debug_set_wait_limit(unsigned long long ns);

/*
 * Diagnostic: waits for the device, then returns in *site (and clears) the
 * record of the first bounded wait of the tensor-core prefill that ran out on
 * the current device since the last read: 0 if none, else bit 31 set, the
 * warp in bits 24-29, the kernel's barrier index in bits 16-23, the awaited
 * phase parity in bit 15 and the CTA index (low 15 bits) in bits 0-14.
 * Returns GDR_OK, GDR_ERR_NULL, GDR_ERR_DEVICE or GDR_ERR_LAUNCH.
 */
int gdr_debug_timeout_site(unsigned int *site);

/*
 * Diagnostic: which schedule of the tensor-core prefill gdr_chunk_fwd_workspace
 * sizes for the calls that follow in this process: 0 by shape (the default), 1
 * always the one-kernel schedule (the query gives 0), 2 always the two-kernel
 * schedule.  Lets the tests compare both schedules on the same inputs.
 * Returns GDR_OK, or GDR_ERR_SHAPE for another value.
 */
int gdr_debug_set_chunk_schedule(int schedule);

/* Static description of a status code; never NULL. */
const char *gdr_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H */
