/*
 * rda.h -- C ABI of the RDA (Raon Delta Attention) core for NVIDIA B200 (sm_100a).
 *
 * WHAT IS COMPUTED
 *   Per sequence and head, the gated delta rule.  The article "Raon-1 nano:
 *   half of a 3.1B model is a lookup table, and a 99M model keeps one too",
 *   section "The other 1.5B: a hybrid built to forget", describes the
 *   reference recurrence: it decays the state, computes the error between the
 *   value and the state's prediction for the key, writes that error with
 *   strength beta, and rescales the value with a separate write gate.  In
 *   matrix form, with the math-orientation state S (Dv x Dk):
 *
 *       S_t = alpha_t * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t (gamma_t v_t) k_t^T
 *       o_t = scale * S_t q_t                       (post-update read)
 *
 *   alpha_t = exp(log_alpha_t) is a scalar per (token, head); gamma_t is the
 *   optional write gate (NULL means 1).  Preconditions, not checked: log_alpha
 *   in [-5, 0] (the article bounds the decay below by -5 in log space),
 *   beta in [0, 1], all inputs finite.  Outside them the result is unspecified
 *   but the call still terminates.
 *
 * STATE
 *   fp32, as the blog post on the Raon-1 mini vLLM pull request lists for its
 *   fast kernels (FP32 recurrent state) and as the nano article sizes it
 *   (16 heads x 128 x 128 fp32 per layer).  Stored as [.., H, Dk, Dv]
 *   row-major: element [i][j] is S[j][i] (i indexes the key dimension, j the
 *   value dimension).
 *
 * LAYOUTS (all row-major, contiguous, no padding)
 *   q, k   [B, T, H, Dk]        (varlen: [total_T, H, Dk])
 *   v, out [B, T, H, Dv]        (varlen: [total_T, H, Dv])
 *   log_alpha, beta, write_gate  fp32 [B, T, H]  (varlen: [total_T, H])
 *   states fp32 [B, H, Dk, Dv]  (varlen: [num_seqs, H, Dk, Dv])
 *   q, k, v and out share one element type, rda_dtype_t.
 *
 * OWNERSHIP AND ORDERING
 *   Every pointer named "device" is device memory owned by the caller; the
 *   library allocates no device memory and keeps no per-call state.  The one
 *   exception is rda_prefill_chunked_noalloc's fixed scratch array, a static
 *   device array of the library (described with that call).  Each call
 *   enqueues its work on `stream` (a cudaStream_t, passed as void*; NULL is the
 *   legacy default stream) and returns without synchronising.  Calls are
 *   thread-safe.  Input buffers must not be modified, and outputs not read,
 *   until the stream has reached the call.  The first call of an entry point
 *   in a process sets kernel attributes (host-side, once); make it outside
 *   stream capture.  Later calls only enqueue kernels, so a CUDA graph
 *   captured from `stream` replays them; the exception is rda_prefill_varlen
 *   (and its per-channel form) with a non-NULL cu_seqlens_host, which copies a
 *   schedule from temporary host memory and must not be captured (pass NULL
 *   under capture).  This paragraph's capture statement does not cover
 *   rda_prefill_chunked_noalloc, which is described with that call.
 *
 * ALIASING
 *   final_state may equal initial_state (updated in place).  No other output
 *   may overlap any input or another output.
 *
 * ERRORS
 *   Argument errors are detected on the host before anything is enqueued and
 *   returned synchronously; nothing is launched then.  A failed launch returns
 *   RDA_ERR_CUDA.  Kernels never trap: a device-side wait that exceeds its
 *   bound records RDA_ERR_TIMEOUT in the workspace error word, stops the
 *   affected work and returns; read it with rda_read_device_error().
 *
 * SUPPORTED SHAPES
 *   Dk, Dv in {64, 128}.  B, T, H >= 0 with B*T*H*max(Dk,Dv) < 2^31 per
 *   tensor.  T = 0 (or B = 0) is a no-op that copies initial to final state.
 */
#ifndef RDA_H_
#define RDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RDA_OK = 0,
    RDA_ERR_INVALID_ARG = 1,   /* null required pointer, negative size, bad cu_seqlens */
    RDA_ERR_UNSUPPORTED = 2,   /* Dk or Dv outside {64, 128}, unknown dtype          */
    RDA_ERR_MISALIGNED = 3,    /* a pointer breaks the 16-byte alignment rule        */
    RDA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required         */
    RDA_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed        */
    RDA_ERR_TIMEOUT = 6        /* a bounded device-side wait ran out                 */
} rda_status_t;

typedef enum {
    RDA_F32 = 0,               /* q, k, v, out are float                             */
    RDA_BF16 = 1               /* q, k, v, out are bfloat16 (raw 16-bit words)       */
} rda_dtype_t;

typedef enum {
    RDA_ACT_NONE = 0,          /* identity                                           */
    RDA_ACT_SILU = 1,          /* x * sigmoid(x)                                     */
    RDA_ACT_SIGMOID = 2        /* 1 / (1 + exp(-x))                                  */
} rda_act_t;

/* Static, human-readable name of a status code.  Never NULL. */
const char *rda_status_string(rda_status_t status);

/* Library version string, e.g. "0.1.0". */
const char *rda_version(void);

/*
 * Bytes of device workspace that rda_prefill_chunked (num_seqs = 0) or
 * rda_prefill_varlen (num_seqs = N, pass B = 1 and T = total_T) needs for
 * these sizes, enough for either dtype.  Always >= 256: the first 256 bytes
 * hold the device error word.  When the chunked tensor-core path can run
 * (Dk = 128) it also holds that path's per-chunk scratch, about 40.5 KiB
 * per 64-token chunk and head at Dv = 128 (e.g. 42 MB for B=1, T=4096, H=16).
 * The workspace must be 256-byte aligned; its contents need no
 * initialisation beyond a cleared error word, and are overwritten by each
 * call.  Returns 0 for unsupported sizes.
 */
size_t rda_prefill_workspace_bytes(int B, int T, int H, int Dk, int Dv, int num_seqs);

/*
 * Fixed-length prefill over B sequences of T tokens each.
 *
 * Defined by the gated delta rule above; the chunked form it uses reaches the
 * same result up to rounding: 64-token chunks, a UT transform of each chunk
 * and its products on the tensor cores, with the chunk-local operands of the
 * outputs (chunk-parallel), then a sequential scan of the fp32 state across
 * chunks that also produces the outputs.  bf16
 * inputs take this path when Dk = 128; fp32 inputs, and bf16 with Dk = 64,
 * take a token-sequential fp32 path (fp32 inputs are held to fp32 accuracy,
 * which bf16 tensor-core operands cannot give).  Several kernels are
 * enqueued on `stream`, in order.
 *
 *   q, k, v        device, dtype, layouts above, 16-byte aligned
 *   log_alpha      device fp32 [B,T,H]; beta device fp32 [B,T,H]
 *   write_gate     device fp32 [B,T,H] or NULL (gamma = 1)
 *   initial_state  device fp32 [B,H,Dk,Dv] or NULL (zero state)
 *   final_state    device fp32 [B,H,Dk,Dv] or NULL (not returned)
 *   out            device, dtype, [B,T,H,Dv], 16-byte aligned
 *   scale          multiplies the output only
 *   workspace      device, >= rda_prefill_workspace_bytes(B,T,H,Dk,Dv,0)
 */
rda_status_t rda_prefill_chunked(const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta,
                                 const float *write_gate,
                                 const float *initial_state, float *final_state,
                                 void *out, rda_dtype_t dtype,
                                 int B, int T, int H, int Dk, int Dv, float scale,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * Variable-length prefill over num_seqs sequences packed along the token axis.
 * Sequence n owns tokens [cu_seqlens[n], cu_seqlens[n+1]); chunks restart at
 * every sequence start and never cross a boundary.  A zero-length sequence
 * copies its initial state to its final state.
 *
 *   cu_seqlens       device int32 [num_seqs+1], non-decreasing, cu_seqlens[0] = 0,
 *                    cu_seqlens[num_seqs] = total_T
 *   cu_seqlens_host  host int32 [num_seqs+1] mirror of cu_seqlens, or NULL.  When
 *                    given, it is validated and used to schedule the longest
 *                    sequences first; it is read before the call returns.
 *   initial_states   device fp32 [num_seqs,H,Dk,Dv] or NULL (zero states)
 *   final_states     device fp32 [num_seqs,H,Dk,Dv] or NULL
 *   other arguments  as rda_prefill_chunked, with B*T replaced by total_T
 *   workspace        device, >= rda_prefill_workspace_bytes(1,total_T,H,Dk,Dv,num_seqs)
 */
rda_status_t rda_prefill_varlen(const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta,
                                const float *write_gate,
                                const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                int num_seqs, int total_T,
                                const float *initial_states, float *final_states,
                                void *out, rda_dtype_t dtype,
                                int H, int Dk, int Dv, float scale,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * One decode step for B independent sequences (one new token each), state
 * updated in place.  It is the T = 1 case of the rule above, evaluated in one
 * pass over the state: with a = S_old k and b = S_old q,
 *   e = gamma v - alpha a,  o = scale (alpha b + beta (k.q) e),
 *   S_new = alpha S_old + beta e k^T.
 *
 *   q, k   device, dtype, [B,H,Dk];  v device, dtype, [B,H,Dv]
 *   log_alpha, beta  device fp32 [B,H];  write_gate device fp32 [B,H] or NULL
 *   state  device fp32 [B,H,Dk,Dv], read and overwritten, 16-byte aligned
 *   out    device, dtype, [B,H,Dv]
 */
rda_status_t rda_decode_step(const void *q, const void *k, const void *v,
                             const float *log_alpha, const float *beta,
                             const float *write_gate,
                             float *state, void *out, rda_dtype_t dtype,
                             int B, int H, int Dk, int Dv, float scale, void *stream);

/*
 * Multi-token decode: T new tokens per sequence (1 <= T <= 8), state updated in
 * place, with the result of T successive rda_decode_step calls (equivalently,
 * a T-token prefill from the state).  For speculative decoding: the model card
 * "KRAFTON/Raon-1-nano-gguf" (section "Model: KRAFTON/Raon-1-nano-gguf") runs
 * multi-token prediction with draft tokens per step, and the blog post on
 * Raon-1 mini (section "Bạn có thể chạy gì trong tuần này") quotes a draft model
 * at block size 8.  The state is read and written once whatever T is: after t
 * tokens every row of the state is a combination of its old value and the new
 * keys, so the kernel needs only the old state's products with the T keys and
 * queries, and the tokens' Gram values.
 *
 *   q, k   device, dtype, [B,T,H,Dk];  v, out device, dtype, [B,T,H,Dv]
 *   log_alpha, beta  device fp32 [B,T,H];  write_gate device fp32 [B,T,H] or NULL
 *   state  device fp32 [B,H,Dk,Dv], read and overwritten, 16-byte aligned
 * Returns RDA_ERR_UNSUPPORTED for T > 8; T = 0 (or B = 0) does nothing.
 */
rda_status_t rda_decode_tokens(const void *q, const void *k, const void *v,
                               const float *log_alpha, const float *beta,
                               const float *write_gate,
                               float *state, void *out, rda_dtype_t dtype,
                               int B, int T, int H, int Dk, int Dv, float scale, void *stream);

/*
 * PER-KEY-CHANNEL DECAY
 *
 * The model printout in the "tiny-random/raon-1-mini" README (section
 * "Printing the model") gives the RDA layer decay projections f_a_proj /
 * f_b_proj whose output is as wide as heads x key dims, and the blog post on
 * Raon-1 mini (architecture section) and the nano article (section "The other
 * 1.5B") describe RDA as a modification of Kimi Delta Attention, whose decay is
 * per key channel.  These three calls take that form: log_alpha holds one
 * decay per key dimension, and key dimension i of the state decays by alpha_i
 * (the same order: decay, error against the decayed state, write, read):
 *
 *     S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t (gamma_t v_t) k_t^T
 *     o_t = scale * S_t q_t
 *
 * With every alpha_t[i] equal this is the scalar rule above.  Arguments,
 * layouts, results and errors are those of the scalar calls except:
 *   log_alpha  device fp32 [B,T,H,Dk] (varlen: [total_T,H,Dk]; decode: [B,H,Dk]),
 *              each value in [-5, 0] (precondition, not checked)
 * The prefill calls take the chunked tensor-core path for bf16 with Dk = 128
 * (the decayed Grams split around a reference token of each 16-token block,
 * and the decayed K and Q of each chunk stored as images next to -W, P and
 * U'), and evaluate the rule token by token in fp32 otherwise (fp32, or
 * Dk = 64).  Their workspace is rda_prefill_channel_workspace_bytes(...) bytes
 * (256-byte aligned; larger than the scalar calls' on the chunked path);
 * RDA_ERR_WORKSPACE when it is missing or smaller.
 */
size_t rda_prefill_channel_workspace_bytes(int B, int T, int H, int Dk, int Dv, int num_seqs);

rda_status_t rda_prefill_chunked_channel(const void *q, const void *k, const void *v,
                                         const float *log_alpha, const float *beta,
                                         const float *write_gate,
                                         const float *initial_state, float *final_state,
                                         void *out, rda_dtype_t dtype,
                                         int B, int T, int H, int Dk, int Dv, float scale,
                                         void *workspace, size_t workspace_bytes, void *stream);

rda_status_t rda_prefill_varlen_channel(const void *q, const void *k, const void *v,
                                        const float *log_alpha, const float *beta,
                                        const float *write_gate,
                                        const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                        int num_seqs, int total_T,
                                        const float *initial_states, float *final_states,
                                        void *out, rda_dtype_t dtype,
                                        int H, int Dk, int Dv, float scale,
                                        void *workspace, size_t workspace_bytes, void *stream);

rda_status_t rda_decode_step_channel(const void *q, const void *k, const void *v,
                                     const float *log_alpha, const float *beta,
                                     const float *write_gate,
                                     float *state, void *out, rda_dtype_t dtype,
                                     int B, int H, int Dk, int Dv, float scale, void *stream);

/*
 * THE STEPS AROUND THE CORE
 *
 * The model printout in the "tiny-random/raon-1-mini" README (section
 * "Printing the model") shows what the RDA layer does before and after the
 * recurrence: q, k and v pass through short convolutions (q_conv1d, k_conv1d,
 * v_conv1d) after their projections; b_proj and rda_w_proj give the write
 * strength and the write gate; g_proj gives an output gate and o_norm, an
 * RMSNorm over the head dimension (eps 1e-5), normalises the core's output.
 * The nano article sizes the per-layer convolution window at three tokens
 * (section "The cache is small if the runtime keeps it small") and gives the
 * write gate sigma(beta_raw + delta) / sigma(beta_raw) and the decay's lower
 * bound of -5 in log space (section "The other 1.5B"); the blog post on Raon-1
 * mini keeps the convolution history in BF16.  Where the pages are silent the
 * reading taken is stated with the argument.
 *
 * rda_prep_inputs: from the projections' outputs to the core's inputs, one
 * pass, per sequence n and token t:
 *   y_t = act(w[c][0] x_{t-2} + w[c][1] x_{t-1} + w[c][2] x_t)  per channel c of
 *         q, k and v (a causal depthwise 3-tap convolution; x_{-1}, x_{-2} come
 *         from the carried window)
 *   q_t, k_t = y_t / ||y_t||_2 per head;  v_t = y_t
 *   beta = sigmoid(beta_raw);  write_gate = sigmoid(beta_raw + delta) / beta
 *   log_alpha = min(max(log_alpha_raw, -5), 0)
 *
 *   q_raw, k_raw   device, dtype, [total_T,H,Dk];  v_raw device, dtype, [total_T,H,Dv]
 *   conv_w_q, conv_w_k  device fp32 [H*Dk, 3];  conv_w_v device fp32 [H*Dv, 3]
 *                  (taps for t-2, t-1, t; channel c = head * D + d)
 *   conv_window_in   device bf16 [num_seqs, 3, H*Dk + H*Dk + H*Dv] or NULL
 *                  (zeros): the last three raw inputs of each sequence before
 *                  this call, oldest first, channels of q, k, v concatenated
 *   conv_window_out  device bf16, same layout, or NULL: the last three raw
 *                  inputs after this call (may equal conv_window_in)
 *   beta_raw       device fp32 [total_T,H];  delta device fp32 [total_T,H] or NULL
 *   log_alpha_raw  device fp32 [total_T,H], or [total_T,H,Dk] with channel_decay != 0
 *   cu_seqlens     device int32 [num_seqs+1] (packed sequences; max_seqlen must
 *                  be at least the longest one), or NULL: num_seqs sequences of
 *                  seq_len tokens (total_T = num_seqs * seq_len)
 *   q, k, v        device, dtype, outputs in the core's layouts
 *   beta, log_alpha  device fp32 outputs like beta_raw, log_alpha_raw
 *   write_gate     device fp32 [total_T,H] output; NULL exactly when delta is NULL
 *   conv_act       RDA_ACT_NONE or RDA_ACT_SILU (the pages do not name the
 *                  convolution's activation; Kimi Delta Attention, which the
 *                  pages say RDA modifies, uses SiLU)
 * q_raw, k_raw, v_raw, q, k, v must be 16-byte aligned.
 */
rda_status_t rda_prep_inputs(const void *q_raw, const void *k_raw, const void *v_raw,
                             const float *conv_w_q, const float *conv_w_k, const float *conv_w_v,
                             const void *conv_window_in, void *conv_window_out,
                             const float *beta_raw, const float *delta,
                             const float *log_alpha_raw, int channel_decay,
                             const int32_t *cu_seqlens, int num_seqs, int seq_len, int max_seqlen, int total_T,
                             void *q, void *k, void *v, float *beta, float *write_gate, float *log_alpha,
                             rda_dtype_t dtype, int H, int Dk, int Dv, rda_act_t conv_act, void *stream);

/*
 * rda_output_gate_norm: after the core, per token and head,
 *   out = o / sqrt(mean_d(o^2) + eps) * norm_weight * act(g)
 *
 *   o, g, out      device, dtype, [tokens,H,Dv], 16-byte aligned (out may equal o)
 *   norm_weight    device fp32 [Dv] (o_norm's weight, shared by the heads)
 *   gate_act       RDA_ACT_SIGMOID, RDA_ACT_SILU or RDA_ACT_NONE (the pages do
 *                  not name the output gate's activation)
 */
rda_status_t rda_output_gate_norm(const void *o, const void *g, const float *norm_weight, float eps,
                                  rda_act_t gate_act, void *out, rda_dtype_t dtype,
                                  long long tokens, int H, int Dv, void *stream);

/*
 * BACKWARD PASS
 *
 * The pages never discuss training; this is the reverse-mode derivative of
 * the rule above (the order of the nano article's section "The other 1.5B":
 * decay, error against the decayed state, write, read), for the loss
 *     L = <d_out, out> + <d_final_state, final_state>
 * of a fixed-length prefill.  Evaluated token by token in fp32: a forward pass
 * stores the state entering every 16-token tile in the workspace, and the
 * backward pass walks the tiles in reverse, recomputing each tile's states from
 * its checkpoint.  Scalar decay per (token, head).
 *
 *   q, k, v, log_alpha, beta, write_gate, initial_state, dtype, B..Dv, scale:
 *                  as rda_prefill_chunked (write_gate and initial_state nullable)
 *   d_out          device, dtype, [B,T,H,Dv]
 *   d_final_state  device fp32 [B,H,Dk,Dv] or NULL (zero)
 *   dq, dk         device fp32 [B,T,H,Dk];  dv device fp32 [B,T,H,Dv]
 *   d_log_alpha, d_beta  device fp32 [B,T,H]
 *   d_write_gate   device fp32 [B,T,H]; NULL exactly when write_gate is NULL
 *   d_initial_state  device fp32 [B,H,Dk,Dv] or NULL (not returned); it is
 *                  also the gradient of a zero initial state when that is NULL
 *   workspace      device, >= rda_backward_workspace_bytes(B,T,H,Dk,Dv)
 *                  (B H ceil(T/16) Dk Dv fp32 checkpoints plus 256 bytes:
 *                  256 MiB for B=1, T=4096, H=16, D=128)
 * Outputs are overwritten (the call clears the summed ones first); none may
 * alias an input.
 */
size_t rda_backward_workspace_bytes(int B, int T, int H, int Dk, int Dv);

rda_status_t rda_backward(const void *q, const void *k, const void *v,
                          const float *log_alpha, const float *beta, const float *write_gate,
                          const float *initial_state, const void *d_out, const float *d_final_state,
                          float *dq, float *dk, float *dv, float *d_log_alpha, float *d_beta,
                          float *d_write_gate, float *d_initial_state,
                          rda_dtype_t dtype, int B, int T, int H, int Dk, int Dv, float scale,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * Fixed-length prefill that allocates nothing and takes no workspace.
 *
 * The pages describe no such call; it exists for callers that cannot give the
 * library scratch memory: host programs that own all device memory themselves
 * (an inference server that sizes its memory pool once at start-up and allows
 * no cudaMalloc afterwards, a plug-in whose host framework passes tensors but
 * offers no way to ask for scratch).  Arguments, layouts and argument errors
 * are those of rda_prefill_chunked, and its results equal that call's bit for
 * bit; it calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Its scratch is a fixed 64 MiB array in device memory that every GPU loading
 * this library holds until the process exits.  A call that needs more scratch
 * than that (rda_prefill_workspace_bytes for bf16 inputs with Dk = 128: about
 * 1,600 chunk-head pairs at Dv = 128, i.e. H = 16 and T up to about 6,400; the
 * nano shape T = 4096, H = 16 fits) is rejected with RDA_ERR_WORKSPACE.  The
 * token-sequential path (fp32 inputs, or Dk = 64) needs only the error word and
 * is never rejected for size.  Like every other argument error, a rejection
 * enqueues nothing.  Each call looks up the array's device address in the
 * current context; the first call in a context also loads the library's device
 * code, so make it before any stream capture.  All calls on a device share the
 * array, which keeps the last call's contents: calls whose work overlaps on the
 * GPU (unordered streams) race on it.  Each accepted call clears the array's
 * device error word before launching; a device-side timeout is not reported
 * back through this call.
 */
rda_status_t rda_prefill_chunked_noalloc(const void *q, const void *k, const void *v,
                                         const float *log_alpha, const float *beta,
                                         const float *write_gate,
                                         const float *initial_state, float *final_state,
                                         void *out, rda_dtype_t dtype,
                                         int B, int T, int H, int Dk, int Dv, float scale,
                                         void *stream);

/*
 * TESTING ONLY: fault injection for the device-side timeout path.
 *
 * Process-wide; affects the prefill calls made after it returns.  The bound of
 * every device-side wait becomes `wait_limit_ns` (0 restores the default, 4 s),
 * and, when drop_chunk >= 0, the state scan of the chunked path never fills
 * the operands of chunk `drop_chunk` of each (sequence, head, value slice):
 * the scan's wait for that chunk runs out, the kernel records RDA_ERR_TIMEOUT
 * in the workspace error word, waits (bounded) for the copies it already has
 * in flight and returns, leaving the outputs from that chunk on and the final
 * state unwritten.  The context stays usable.  rda_debug_set_wait_fault(-1, 0)
 * turns it off (the default).  Not for production use: no other argument is
 * checked, and calls on other threads see the setting too.
 */
void rda_debug_set_wait_fault(int drop_chunk, unsigned long long wait_limit_ns);

/*
 * Waits for `stream`, then reads and clears the device error word at the start
 * of `workspace`.  Writes RDA_OK or the recorded code to *code.  Returns
 * RDA_ERR_CUDA if the copy fails.
 */
rda_status_t rda_read_device_error(void *workspace, int *code, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RDA_H_ */
