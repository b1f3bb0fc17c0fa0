// Internal launch interface shared by the C-ABI layer and the kernels.
// Not installed; the public interface is include/rda.h.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "rda.h"

namespace rda {

// Device error word: first 4 bytes of the caller's workspace.
constexpr size_t kErrorWordBytes = 256;

// Arguments common to every prefill launch.  Token rows are addressed as
// (global token index) * H + head; fixed-length batches use seq_start = b * T,
// packed batches read cu_seqlens.
struct PrefillArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *gamma;
    const float *s0;
    float *sf;
    void *out;
    const int32_t *cu_seqlens;   // null for fixed-length batches
    const int32_t *order;        // optional schedule: sequence index per grid z, or null
    int num_seqs;                // B (fixed) or N (packed)
    int T;                       // tokens per sequence (fixed only)
    int total_T;                 // B*T or packed total
    int H, Dk, Dv;
    float scale;
    int32_t *err;                // device error word
    uint64_t wait_ns;            // bound of every device-side wait
    int debug_drop_chunk;        // fault injection (tests only): the scan never fills this chunk; -1 = off
    bool channel_decay;          // log_alpha is per key channel: [tokens, H, Dk]
    float *ckpt;                 // token-sequential path: the state entering every 16-token tile, or null
    // chunked path only (filled by launch_chunked)
    const int32_t *chunk_base;   // packed: first global chunk of each sequence [N+1]
    uint8_t *workspace_chunks;   // per (chunk, head) prep results
    size_t chunk_bytes;          // bytes per (chunk, head)
};

struct DecodeArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *gamma;
    float *state;
    void *out;
    int B, H, Dk, Dv;
    float scale;
    int T;                       // tokens per sequence (multi-token decode only)
    bool channel_decay;          // log_alpha is per key channel: [B, H, Dk]
};

// Bound of the device-side waits, and the test-only fault injection, as set by
// rda_debug_set_wait_fault (defaults: 4 s, no fault).
struct WaitSettings {
    uint64_t wait_ns;
    int drop_chunk;
};
WaitSettings wait_settings();

// The steps around the core (rda_prep_inputs, rda_output_gate_norm).
struct PrepLaunch {
    const void *raw[3];          // q, k, v projections
    const float *w[3];           // conv taps [H*D, 3]
    const void *win_in;          // bf16 [N, 3, C] or null (zeros)
    void *win_out;               // bf16 [N, 3, C] or null
    const float *beta_raw, *delta, *la_raw;
    const int32_t *cu_seqlens;   // null: num_seqs sequences of seq_len tokens
    int num_seqs, seq_len, max_seqlen, H, Dk, Dv;
    bool channel;
    int act;
    rda_dtype_t dtype;
    void *out[3];
    float *beta, *gamma, *log_alpha;
};
cudaError_t launch_prep_inputs(const PrepLaunch &l, cudaStream_t s);
cudaError_t launch_output_gate_norm(const void *o, const void *g, const float *w, void *out, long rows, int Dv,
                                    float eps, int act, rda_dtype_t dtype, cudaStream_t s);

// Backward pass (rda_backward): gradients of <d_out, out> + <d_sf, final state>.
struct BackwardArgs {
    const void *q, *k, *v, *d_out;
    const float *log_alpha, *beta, *gamma, *d_sf;
    const float *ckpt;           // states entering every 16-token tile, [B][H][tiles][Dk][Dv]
    float *dq, *dk, *dv, *d_log_alpha, *d_beta, *d_gamma, *d_s0;
    int B, T, H, Dk, Dv;
    float scale;
};
cudaError_t launch_backward(const BackwardArgs &a, rda_dtype_t dtype, cudaStream_t s);
size_t backward_ckpt_bytes(int B, int T, int H, int Dk, int Dv);

// Most tokens one multi-token decode call takes per sequence.
constexpr int kMaxDecodeTokens = 8;

cudaError_t launch_recurrent(const PrefillArgs &a, rda_dtype_t dtype, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs &a, rda_dtype_t dtype, cudaStream_t s);
cudaError_t launch_decode_tokens(const DecodeArgs &a, rda_dtype_t dtype, cudaStream_t s);
// Chunked tensor-core prefill (bf16, Dk = 128, Dv in {64, 128}).  `scratch`
// points at chunked_workspace_bytes() bytes of device memory (256-aligned).
cudaError_t launch_chunked(const PrefillArgs &a, void *scratch, cudaStream_t s);
bool chunked_supported(rda_dtype_t dtype, int Dk, int Dv);
// Scratch the chunked path needs: fixed-length batches pass num_seqs = 0.
size_t chunked_workspace_bytes(long total_T, int T, int B, int H, int Dv, int num_seqs, bool channel = false);

// Host-side argument checks of rda_prefill_chunked except those of the
// workspace; enqueues nothing.  On RDA_OK, *scratch_bytes is the workspace
// that call needs for these arguments (the error word alone on the
// token-sequential path).  `channel`: per-key-channel log alpha [.., T, H, Dk].
rda_status_t validate_prefill_chunked(const void *q, const void *k, const void *v, const float *log_alpha,
                                      const float *beta, const float *write_gate, const float *initial_state,
                                      const float *final_state, const void *out, rda_dtype_t dtype, int B,
                                      int T, int H, int Dk, int Dv, size_t *scratch_bytes, bool channel = false);

}  // namespace rda
