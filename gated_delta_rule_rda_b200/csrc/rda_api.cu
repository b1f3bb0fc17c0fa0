// C-ABI entry points (include/rda.h): argument validation on the host, then
// dispatch to the kernels on the caller's stream.  Nothing here allocates
// device memory; nothing here computes any part of the recurrence.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <numeric>
#include <vector>

#include "rda_internal.h"

using namespace rda;

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool dims_ok(int Dk, int Dv) { return (Dk == 64 || Dk == 128) && (Dv == 64 || Dv == 128); }

// Largest element count of any one tensor must stay below 2^31.
bool sizes_ok(long long tokens, int H, int Dk, int Dv) {
    const long long m = tokens * H * std::max(Dk, Dv);
    return tokens >= 0 && H > 0 && m < (1LL << 31);
}

rda_status_t check_io_ptrs(const void *q, const void *k, const void *v, const float *la,
                           const float *be, const void *out) {
    if (!q || !k || !v || !la || !be || !out) return RDA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return RDA_ERR_MISALIGNED;
    if (!aligned(la, 4) || !aligned(be, 4)) return RDA_ERR_MISALIGNED;
    return RDA_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout: [0, 256) error word; then, for packed batches, the
// longest-first schedule (int32 per sequence); then, when the chunked
// tensor-core path can run (Dk = 128), its per-chunk prep scratch (larger
// with a decay per key dim: the decayed K and Q images go there too).
size_t order_bytes(int num_seqs) { return num_seqs > 0 ? align_up(sizeof(int32_t) * (size_t)num_seqs, 256) : 0; }

size_t workspace_bytes(int B, long T, int H, int Dk, int Dv, int num_seqs, bool channel = false) {
    size_t b = kErrorWordBytes + order_bytes(num_seqs);
    if (chunked_supported(RDA_BF16, Dk, Dv))
        b += align_up(chunked_workspace_bytes(num_seqs > 0 ? T : (long)B * T, (int)T, B, H, Dv, num_seqs, channel),
                      256);
    return b;
}

}  // namespace

namespace rda {

namespace {
constexpr uint64_t kDefaultWaitNs = 4000000000ull;   // 4 s
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
std::atomic<int> g_drop_chunk{-1};
}  // namespace

WaitSettings wait_settings() { return WaitSettings{g_wait_ns.load(), g_drop_chunk.load()}; }

rda_status_t validate_prefill_chunked(const void *q, const void *k, const void *v, const float *log_alpha,
                                      const float *beta, const float *write_gate, const float *initial_state,
                                      const float *final_state, const void *out, rda_dtype_t dtype, int B,
                                      int T, int H, int Dk, int Dv, size_t *scratch_bytes, bool channel) {
    if (dtype != RDA_F32 && dtype != RDA_BF16) return RDA_ERR_UNSUPPORTED;
    if (B < 0 || T < 0 || H <= 0) return RDA_ERR_INVALID_ARG;
    if (!dims_ok(Dk, Dv)) return RDA_ERR_UNSUPPORTED;
    if (!sizes_ok((long long)B * T, H, Dk, Dv)) return RDA_ERR_INVALID_ARG;
    if ((long long)B * H * Dk * Dv >= (1LL << 31)) return RDA_ERR_INVALID_ARG;
    if ((initial_state && !aligned(initial_state, 16)) || (final_state && !aligned(final_state, 16)))
        return RDA_ERR_MISALIGNED;
    if (write_gate && !aligned(write_gate, 4)) return RDA_ERR_MISALIGNED;
    if (B > 0 && T > 0) {
        rda_status_t st = check_io_ptrs(q, k, v, log_alpha, beta, out);
        if (st != RDA_OK) return st;
    }
    *scratch_bytes = chunked_supported(dtype, Dk, Dv) ? workspace_bytes(B, T, H, Dk, Dv, 0, channel)
                                                      : kErrorWordBytes;
    return RDA_OK;
}

}  // namespace rda

extern "C" {

const char *rda_status_string(rda_status_t s) {
    switch (s) {
        case RDA_OK: return "RDA_OK";
        case RDA_ERR_INVALID_ARG: return "RDA_ERR_INVALID_ARG: null required pointer, negative size or bad cu_seqlens";
        case RDA_ERR_UNSUPPORTED: return "RDA_ERR_UNSUPPORTED: Dk and Dv must be 64 or 128; dtype must be RDA_F32 or RDA_BF16";
        case RDA_ERR_MISALIGNED: return "RDA_ERR_MISALIGNED: q, k, v, out, state and workspace must be 16-byte aligned (workspace 256)";
        case RDA_ERR_WORKSPACE: return "RDA_ERR_WORKSPACE: workspace missing or smaller than rda_prefill_workspace_bytes()";
        case RDA_ERR_CUDA: return "RDA_ERR_CUDA: a CUDA runtime call or kernel launch failed";
        case RDA_ERR_TIMEOUT: return "RDA_ERR_TIMEOUT: a bounded device-side wait ran out";
    }
    return "RDA_ERR_UNKNOWN";
}

const char *rda_version(void) { return "0.1.0"; }

size_t rda_prefill_workspace_bytes(int B, int T, int H, int Dk, int Dv, int num_seqs) {
    if (B < 0 || T < 0 || H <= 0 || num_seqs < 0 || !dims_ok(Dk, Dv)) return 0;
    return workspace_bytes(B, T, H, Dk, Dv, num_seqs);
}

size_t rda_prefill_channel_workspace_bytes(int B, int T, int H, int Dk, int Dv, int num_seqs) {
    if (B < 0 || T < 0 || H <= 0 || num_seqs < 0 || !dims_ok(Dk, Dv)) return 0;
    return workspace_bytes(B, T, H, Dk, Dv, num_seqs, true);
}

static rda_status_t prefill_chunked_impl(bool channel, const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta,
                                 const float *write_gate,
                                 const float *initial_state, float *final_state,
                                 void *out, rda_dtype_t dtype,
                                 int B, int T, int H, int Dk, int Dv, float scale,
                                 void *workspace, size_t workspace_bytes_given, void *stream) {
    size_t need = 0;
    rda_status_t st = validate_prefill_chunked(q, k, v, log_alpha, beta, write_gate, initial_state, final_state,
                                               out, dtype, B, T, H, Dk, Dv, &need, channel);
    if (st != RDA_OK) return st;
    if (!workspace || workspace_bytes_given < need) return RDA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return RDA_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (B == 0 || T == 0) {
        if (B > 0 && final_state) {
            const size_t bytes = sizeof(float) * (size_t)B * H * Dk * Dv;
            cudaError_t e = initial_state
                ? (initial_state == final_state ? cudaSuccess
                   : cudaMemcpyAsync(final_state, initial_state, bytes, cudaMemcpyDeviceToDevice, s))
                : cudaMemsetAsync(final_state, 0, bytes, s);
            if (e != cudaSuccess) return RDA_ERR_CUDA;
        }
        return RDA_OK;
    }
    PrefillArgs a{};
    a.q = q; a.k = k; a.v = v;
    a.log_alpha = log_alpha; a.beta = beta; a.gamma = write_gate;
    a.s0 = initial_state; a.sf = final_state; a.out = out;
    a.cu_seqlens = nullptr; a.order = nullptr;
    a.num_seqs = B; a.T = T; a.total_T = B * T;
    a.H = H; a.Dk = Dk; a.Dv = Dv; a.scale = scale;
    a.err = static_cast<int32_t *>(workspace);
    const WaitSettings ws = wait_settings();
    a.wait_ns = ws.wait_ns;
    a.debug_drop_chunk = ws.drop_chunk;
    a.channel_decay = channel;
    cudaError_t e = chunked_supported(dtype, Dk, Dv)
                        ? launch_chunked(a, static_cast<char *>(workspace) + kErrorWordBytes, s)
                        : launch_recurrent(a, dtype, s);
    return e == cudaSuccess ? RDA_OK : RDA_ERR_CUDA;
}

rda_status_t rda_prefill_chunked(const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta,
                                 const float *write_gate,
                                 const float *initial_state, float *final_state,
                                 void *out, rda_dtype_t dtype,
                                 int B, int T, int H, int Dk, int Dv, float scale,
                                 void *workspace, size_t workspace_bytes_given, void *stream) {
    return prefill_chunked_impl(false, q, k, v, log_alpha, beta, write_gate, initial_state, final_state, out,
                                dtype, B, T, H, Dk, Dv, scale, workspace, workspace_bytes_given, stream);
}

rda_status_t rda_prefill_chunked_channel(const void *q, const void *k, const void *v,
                                         const float *log_alpha, const float *beta,
                                         const float *write_gate,
                                         const float *initial_state, float *final_state,
                                         void *out, rda_dtype_t dtype,
                                         int B, int T, int H, int Dk, int Dv, float scale,
                                         void *workspace, size_t workspace_bytes_given, void *stream) {
    return prefill_chunked_impl(true, q, k, v, log_alpha, beta, write_gate, initial_state, final_state, out,
                                dtype, B, T, H, Dk, Dv, scale, workspace, workspace_bytes_given, stream);
}

static rda_status_t prefill_varlen_impl(bool channel, const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta,
                                const float *write_gate,
                                const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                int num_seqs, int total_T,
                                const float *initial_states, float *final_states,
                                void *out, rda_dtype_t dtype,
                                int H, int Dk, int Dv, float scale,
                                void *workspace, size_t workspace_bytes_given, void *stream) {
    if (dtype != RDA_F32 && dtype != RDA_BF16) return RDA_ERR_UNSUPPORTED;
    if (num_seqs < 0 || total_T < 0 || H <= 0) return RDA_ERR_INVALID_ARG;
    if (!dims_ok(Dk, Dv)) return RDA_ERR_UNSUPPORTED;
    if (!sizes_ok(total_T, H, Dk, Dv)) return RDA_ERR_INVALID_ARG;
    if ((long long)num_seqs * H * Dk * Dv >= (1LL << 31)) return RDA_ERR_INVALID_ARG;
    if (num_seqs > 0 && !cu_seqlens) return RDA_ERR_INVALID_ARG;
    const bool chunked = chunked_supported(dtype, Dk, Dv);
    const size_t need = chunked ? workspace_bytes(1, total_T, H, Dk, Dv, num_seqs, channel)
                                : kErrorWordBytes + order_bytes(num_seqs);
    if (!workspace || workspace_bytes_given < need) return RDA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return RDA_ERR_MISALIGNED;
    if ((initial_states && !aligned(initial_states, 16)) || (final_states && !aligned(final_states, 16)))
        return RDA_ERR_MISALIGNED;
    if (cu_seqlens && !aligned(cu_seqlens, 4)) return RDA_ERR_MISALIGNED;
    if (total_T > 0) {
        rda_status_t st = check_io_ptrs(q, k, v, log_alpha, beta, out);
        if (st != RDA_OK) return st;
    }
    if (write_gate && !aligned(write_gate, 4)) return RDA_ERR_MISALIGNED;
    if (num_seqs == 0) return RDA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    int32_t *order = nullptr;
    if (cu_seqlens_host) {
        if (cu_seqlens_host[0] != 0 || cu_seqlens_host[num_seqs] != total_T) return RDA_ERR_INVALID_ARG;
        for (int n = 0; n < num_seqs; ++n)
            if (cu_seqlens_host[n + 1] < cu_seqlens_host[n]) return RDA_ERR_INVALID_ARG;
        // Longest sequences first, so that the long tails start early.
        std::vector<int32_t> perm(num_seqs);
        std::iota(perm.begin(), perm.end(), 0);
        std::stable_sort(perm.begin(), perm.end(), [&](int32_t x, int32_t y) {
            return cu_seqlens_host[x + 1] - cu_seqlens_host[x] > cu_seqlens_host[y + 1] - cu_seqlens_host[y];
        });
        order = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + kErrorWordBytes);
        // Pageable source: the copy is staged before cudaMemcpyAsync returns.
        if (cudaMemcpyAsync(order, perm.data(), sizeof(int32_t) * num_seqs, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return RDA_ERR_CUDA;
    }
    PrefillArgs a{};
    a.q = q; a.k = k; a.v = v;
    a.log_alpha = log_alpha; a.beta = beta; a.gamma = write_gate;
    a.s0 = initial_states; a.sf = final_states; a.out = out;
    a.cu_seqlens = cu_seqlens; a.order = order;
    a.num_seqs = num_seqs; a.T = 0; a.total_T = total_T;
    a.H = H; a.Dk = Dk; a.Dv = Dv; a.scale = scale;
    a.err = static_cast<int32_t *>(workspace);
    const WaitSettings ws = wait_settings();
    a.wait_ns = ws.wait_ns;
    a.debug_drop_chunk = ws.drop_chunk;
    a.channel_decay = channel;
    cudaError_t e = chunked
        ? launch_chunked(a, static_cast<char *>(workspace) + kErrorWordBytes + order_bytes(num_seqs), s)
        : launch_recurrent(a, dtype, s);
    return e == cudaSuccess ? RDA_OK : RDA_ERR_CUDA;
}

rda_status_t rda_prefill_varlen(const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta,
                                const float *write_gate,
                                const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                int num_seqs, int total_T,
                                const float *initial_states, float *final_states,
                                void *out, rda_dtype_t dtype,
                                int H, int Dk, int Dv, float scale,
                                void *workspace, size_t workspace_bytes_given, void *stream) {
    return prefill_varlen_impl(false, q, k, v, log_alpha, beta, write_gate, cu_seqlens, cu_seqlens_host, num_seqs,
                               total_T, initial_states, final_states, out, dtype, H, Dk, Dv, scale, workspace,
                               workspace_bytes_given, stream);
}

rda_status_t rda_prefill_varlen_channel(const void *q, const void *k, const void *v,
                                        const float *log_alpha, const float *beta,
                                        const float *write_gate,
                                        const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                        int num_seqs, int total_T,
                                        const float *initial_states, float *final_states,
                                        void *out, rda_dtype_t dtype,
                                        int H, int Dk, int Dv, float scale,
                                        void *workspace, size_t workspace_bytes_given, void *stream) {
    return prefill_varlen_impl(true, q, k, v, log_alpha, beta, write_gate, cu_seqlens, cu_seqlens_host, num_seqs,
                               total_T, initial_states, final_states, out, dtype, H, Dk, Dv, scale, workspace,
                               workspace_bytes_given, stream);
}

static rda_status_t decode_step_impl(bool channel, const void *q, const void *k, const void *v,
                             const float *log_alpha, const float *beta,
                             const float *write_gate,
                             float *state, void *out, rda_dtype_t dtype,
                             int B, int H, int Dk, int Dv, float scale, void *stream) {
    if (dtype != RDA_F32 && dtype != RDA_BF16) return RDA_ERR_UNSUPPORTED;
    if (B < 0 || H <= 0) return RDA_ERR_INVALID_ARG;
    if (!dims_ok(Dk, Dv)) return RDA_ERR_UNSUPPORTED;
    if ((long long)B * H * Dk * Dv >= (1LL << 31)) return RDA_ERR_INVALID_ARG;
    if (B == 0) return RDA_OK;
    rda_status_t st = check_io_ptrs(q, k, v, log_alpha, beta, out);
    if (st != RDA_OK) return st;
    if (!state) return RDA_ERR_INVALID_ARG;
    if (!aligned(state, 16)) return RDA_ERR_MISALIGNED;
    if (write_gate && !aligned(write_gate, 4)) return RDA_ERR_MISALIGNED;
    DecodeArgs a{};
    a.q = q; a.k = k; a.v = v;
    a.log_alpha = log_alpha; a.beta = beta; a.gamma = write_gate;
    a.state = state; a.out = out;
    a.B = B; a.H = H; a.Dk = Dk; a.Dv = Dv; a.scale = scale;
    a.channel_decay = channel;
    return launch_decode(a, dtype, static_cast<cudaStream_t>(stream)) == cudaSuccess ? RDA_OK : RDA_ERR_CUDA;
}

rda_status_t rda_decode_step(const void *q, const void *k, const void *v,
                             const float *log_alpha, const float *beta,
                             const float *write_gate,
                             float *state, void *out, rda_dtype_t dtype,
                             int B, int H, int Dk, int Dv, float scale, void *stream) {
    return decode_step_impl(false, q, k, v, log_alpha, beta, write_gate, state, out, dtype, B, H, Dk, Dv, scale,
                            stream);
}

rda_status_t rda_decode_step_channel(const void *q, const void *k, const void *v,
                                     const float *log_alpha, const float *beta,
                                     const float *write_gate,
                                     float *state, void *out, rda_dtype_t dtype,
                                     int B, int H, int Dk, int Dv, float scale, void *stream) {
    return decode_step_impl(true, q, k, v, log_alpha, beta, write_gate, state, out, dtype, B, H, Dk, Dv, scale,
                            stream);
}

rda_status_t rda_decode_tokens(const void *q, const void *k, const void *v,
                               const float *log_alpha, const float *beta,
                               const float *write_gate,
                               float *state, void *out, rda_dtype_t dtype,
                               int B, int T, int H, int Dk, int Dv, float scale, void *stream) {
    if (dtype != RDA_F32 && dtype != RDA_BF16) return RDA_ERR_UNSUPPORTED;
    if (B < 0 || H <= 0 || T < 0) return RDA_ERR_INVALID_ARG;
    if (T > kMaxDecodeTokens) return RDA_ERR_UNSUPPORTED;
    if (!dims_ok(Dk, Dv)) return RDA_ERR_UNSUPPORTED;
    if ((long long)B * H * Dk * Dv >= (1LL << 31) || (long long)B * T * H * (Dk > Dv ? Dk : Dv) >= (1LL << 31))
        return RDA_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return RDA_OK;
    rda_status_t st = check_io_ptrs(q, k, v, log_alpha, beta, out);
    if (st != RDA_OK) return st;
    if (!state) return RDA_ERR_INVALID_ARG;
    if (!aligned(state, 16)) return RDA_ERR_MISALIGNED;
    if (write_gate && !aligned(write_gate, 4)) return RDA_ERR_MISALIGNED;
    DecodeArgs a{};
    a.q = q; a.k = k; a.v = v;
    a.log_alpha = log_alpha; a.beta = beta; a.gamma = write_gate;
    a.state = state; a.out = out;
    a.B = B; a.T = T; a.H = H; a.Dk = Dk; a.Dv = Dv; a.scale = scale;
    return launch_decode_tokens(a, dtype, static_cast<cudaStream_t>(stream)) == cudaSuccess ? RDA_OK
                                                                                              : RDA_ERR_CUDA;
}

rda_status_t rda_prep_inputs(const void *q_raw, const void *k_raw, const void *v_raw,
                             const float *conv_w_q, const float *conv_w_k, const float *conv_w_v,
                             const void *conv_window_in, void *conv_window_out,
                             const float *beta_raw, const float *delta,
                             const float *log_alpha_raw, int channel_decay,
                             const int32_t *cu_seqlens, int num_seqs, int seq_len, int max_seqlen, int total_T,
                             void *q, void *k, void *v, float *beta, float *write_gate, float *log_alpha,
                             rda_dtype_t dtype, int H, int Dk, int Dv, rda_act_t conv_act, void *stream) {
    if (dtype != RDA_F32 && dtype != RDA_BF16) return RDA_ERR_UNSUPPORTED;
    if (!dims_ok(Dk, Dv)) return RDA_ERR_UNSUPPORTED;
    if (conv_act != RDA_ACT_NONE && conv_act != RDA_ACT_SILU) return RDA_ERR_UNSUPPORTED;
    if (num_seqs < 0 || total_T < 0 || H <= 0 || max_seqlen < 0) return RDA_ERR_INVALID_ARG;
    if (!cu_seqlens && (seq_len < 0 || (long long)num_seqs * seq_len != total_T)) return RDA_ERR_INVALID_ARG;
    if (!sizes_ok(total_T, H, Dk, Dv)) return RDA_ERR_INVALID_ARG;
    if ((long long)num_seqs * 3 * H * (2 * Dk + Dv) >= (1LL << 31)) return RDA_ERR_INVALID_ARG;
    if ((delta == nullptr) != (write_gate == nullptr)) return RDA_ERR_INVALID_ARG;
    if (num_seqs == 0) return RDA_OK;
    if (!conv_w_q || !conv_w_k || !conv_w_v || !beta_raw || !log_alpha_raw || !beta || !log_alpha)
        return RDA_ERR_INVALID_ARG;
    if (total_T > 0) {
        rda_status_t st = check_io_ptrs(q_raw, k_raw, v_raw, beta_raw, log_alpha_raw, q);
        if (st != RDA_OK) return st;
        if (!k || !v) return RDA_ERR_INVALID_ARG;
        if (!aligned(k, 16) || !aligned(v, 16)) return RDA_ERR_MISALIGNED;
    }
    if ((conv_window_in && !aligned(conv_window_in, 2)) || (conv_window_out && !aligned(conv_window_out, 2)))
        return RDA_ERR_MISALIGNED;
    PrepLaunch l{};
    l.raw[0] = q_raw; l.raw[1] = k_raw; l.raw[2] = v_raw;
    l.w[0] = conv_w_q; l.w[1] = conv_w_k; l.w[2] = conv_w_v;
    l.win_in = conv_window_in; l.win_out = conv_window_out;
    l.beta_raw = beta_raw; l.delta = delta; l.la_raw = log_alpha_raw;
    l.cu_seqlens = cu_seqlens;
    l.num_seqs = num_seqs; l.seq_len = seq_len; l.max_seqlen = cu_seqlens ? max_seqlen : seq_len;
    l.H = H; l.Dk = Dk; l.Dv = Dv;
    l.channel = channel_decay != 0; l.act = conv_act; l.dtype = dtype;
    l.out[0] = q; l.out[1] = k; l.out[2] = v;
    l.beta = beta; l.gamma = write_gate; l.log_alpha = log_alpha;
    return launch_prep_inputs(l, static_cast<cudaStream_t>(stream)) == cudaSuccess ? RDA_OK : RDA_ERR_CUDA;
}

rda_status_t rda_output_gate_norm(const void *o, const void *g, const float *norm_weight, float eps,
                                  rda_act_t gate_act, void *out, rda_dtype_t dtype,
                                  long long tokens, int H, int Dv, void *stream) {
    if (dtype != RDA_F32 && dtype != RDA_BF16) return RDA_ERR_UNSUPPORTED;
    if (Dv != 64 && Dv != 128) return RDA_ERR_UNSUPPORTED;
    if (gate_act != RDA_ACT_SIGMOID && gate_act != RDA_ACT_SILU && gate_act != RDA_ACT_NONE)
        return RDA_ERR_UNSUPPORTED;
    if (tokens < 0 || H <= 0 || !(eps >= 0.f)) return RDA_ERR_INVALID_ARG;
    if (tokens * H * Dv >= (1LL << 31)) return RDA_ERR_INVALID_ARG;
    if (tokens == 0) return RDA_OK;
    if (!o || !g || !norm_weight || !out) return RDA_ERR_INVALID_ARG;
    if (!aligned(o, 16) || !aligned(g, 16) || !aligned(out, 16) || !aligned(norm_weight, 4))
        return RDA_ERR_MISALIGNED;
    return launch_output_gate_norm(o, g, norm_weight, out, (long)tokens * H, Dv, eps, gate_act, dtype,
                                   static_cast<cudaStream_t>(stream)) == cudaSuccess ? RDA_OK : RDA_ERR_CUDA;
}

size_t rda_backward_workspace_bytes(int B, int T, int H, int Dk, int Dv) {
    if (B < 0 || T < 0 || H <= 0 || !dims_ok(Dk, Dv)) return 0;
    return kErrorWordBytes + align_up(backward_ckpt_bytes(B, T, H, Dk, Dv), 256);
}

rda_status_t rda_backward(const void *q, const void *k, const void *v,
                          const float *log_alpha, const float *beta, const float *write_gate,
                          const float *initial_state, const void *d_out, const float *d_final_state,
                          float *dq, float *dk, float *dv, float *d_log_alpha, float *d_beta,
                          float *d_write_gate, float *d_initial_state,
                          rda_dtype_t dtype, int B, int T, int H, int Dk, int Dv, float scale,
                          void *workspace, size_t workspace_bytes_given, void *stream) {
    if (dtype != RDA_F32 && dtype != RDA_BF16) return RDA_ERR_UNSUPPORTED;
    if (B < 0 || T < 0 || H <= 0) return RDA_ERR_INVALID_ARG;
    if (!dims_ok(Dk, Dv)) return RDA_ERR_UNSUPPORTED;
    if (!sizes_ok((long long)B * T, H, Dk, Dv)) return RDA_ERR_INVALID_ARG;
    if ((long long)B * H * Dk * Dv >= (1LL << 31)) return RDA_ERR_INVALID_ARG;
    if ((write_gate == nullptr) != (d_write_gate == nullptr)) return RDA_ERR_INVALID_ARG;
    if ((initial_state && !aligned(initial_state, 16)) || (d_final_state && !aligned(d_final_state, 16)) ||
        (d_initial_state && !aligned(d_initial_state, 16)))
        return RDA_ERR_MISALIGNED;
    const size_t need = rda_backward_workspace_bytes(B, T, H, Dk, Dv);
    if (!workspace || workspace_bytes_given < need) return RDA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return RDA_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (B == 0) return RDA_OK;
    if (T == 0) {
        if (d_initial_state) {
            const size_t bytes = sizeof(float) * (size_t)B * H * Dk * Dv;
            cudaError_t e = d_final_state ? cudaMemcpyAsync(d_initial_state, d_final_state, bytes,
                                                            cudaMemcpyDeviceToDevice, s)
                                          : cudaMemsetAsync(d_initial_state, 0, bytes, s);
            if (e != cudaSuccess) return RDA_ERR_CUDA;
        }
        return RDA_OK;
    }
    rda_status_t st = check_io_ptrs(q, k, v, log_alpha, beta, d_out);
    if (st != RDA_OK) return st;
    if (!dq || !dk || !dv || !d_log_alpha || !d_beta) return RDA_ERR_INVALID_ARG;
    if (!aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16)) return RDA_ERR_MISALIGNED;
    // the outputs that collect sums over CTAs start at zero
    const size_t tok = (size_t)B * T * H;
    if (cudaMemsetAsync(dq, 0, tok * Dk * sizeof(float), s) != cudaSuccess ||
        cudaMemsetAsync(dk, 0, tok * Dk * sizeof(float), s) != cudaSuccess ||
        cudaMemsetAsync(d_log_alpha, 0, tok * sizeof(float), s) != cudaSuccess ||
        cudaMemsetAsync(d_beta, 0, tok * sizeof(float), s) != cudaSuccess ||
        (d_write_gate && cudaMemsetAsync(d_write_gate, 0, tok * sizeof(float), s) != cudaSuccess))
        return RDA_ERR_CUDA;
    float *ckpt = reinterpret_cast<float *>(static_cast<char *>(workspace) + kErrorWordBytes);
    // forward pass: the checkpoints (outputs and final state not written)
    PrefillArgs f{};
    f.q = q; f.k = k; f.v = v;
    f.log_alpha = log_alpha; f.beta = beta; f.gamma = write_gate;
    f.s0 = initial_state; f.sf = nullptr; f.out = nullptr;
    f.num_seqs = B; f.T = T; f.total_T = B * T;
    f.H = H; f.Dk = Dk; f.Dv = Dv; f.scale = scale;
    f.err = static_cast<int32_t *>(workspace);
    f.ckpt = ckpt;
    if (launch_recurrent(f, dtype, s) != cudaSuccess) return RDA_ERR_CUDA;
    BackwardArgs b{};
    b.q = q; b.k = k; b.v = v; b.d_out = d_out;
    b.log_alpha = log_alpha; b.beta = beta; b.gamma = write_gate; b.d_sf = d_final_state;
    b.ckpt = ckpt;
    b.dq = dq; b.dk = dk; b.dv = dv; b.d_log_alpha = d_log_alpha; b.d_beta = d_beta;
    b.d_gamma = d_write_gate; b.d_s0 = d_initial_state;
    b.B = B; b.T = T; b.H = H; b.Dk = Dk; b.Dv = Dv; b.scale = scale;
    return launch_backward(b, dtype, s) == cudaSuccess ? RDA_OK : RDA_ERR_CUDA;
}

void rda_debug_set_wait_fault(int drop_chunk, unsigned long long wait_limit_ns) {
    rda::g_drop_chunk.store(drop_chunk < 0 ? -1 : drop_chunk);
    rda::g_wait_ns.store(wait_limit_ns ? (uint64_t)wait_limit_ns : rda::kDefaultWaitNs);
}

rda_status_t rda_read_device_error(void *workspace, int *code, void *stream) {
    if (!workspace || !code) return RDA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t host = 0;
    if (cudaMemcpyAsync(&host, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return RDA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return RDA_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), s) != cudaSuccess) return RDA_ERR_CUDA;
    *code = host;
    return RDA_OK;
}

}  // extern "C"
