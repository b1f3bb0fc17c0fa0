// The steps either side of the RDA core, fused into one kernel each.
//
// Before the core (tiny-random/raon-1-mini README, "Printing the model": q, k
// and v pass through short convolutions after their projections; the nano
// article, "The cache is small if the runtime keeps it small": a three-token
// convolution window per layer; "The other 1.5B": beta, the write gate
// sigma(beta_raw + delta) / sigma(beta_raw), the decay bounded below by -5 in
// log space; the Raon-1 mini blog post: BF16 convolution history):
//
//   y_t = act(w0 x_{t-2} + w1 x_{t-1} + w2 x_t)   per channel of q, k and v
//   q, k <- y / ||y||_2 per head;  v <- y
//   beta = sigmoid(beta_raw),  gamma = sigmoid(beta_raw + delta) / beta,
//   log alpha = clamp(log_alpha_raw, -5, 0)
//
// and the window of the last three raw inputs per channel (bf16) carried
// across calls.  After the core (README: o_norm, an RMSNorm over the head
// dimension, and the output gate g_proj):
//
//   out = o / sqrt(mean(o^2) + eps) * w_norm * act(g)
//
// Both are bound by HBM: each token-head is read and written once.
#include <cuda_bf16.h>

#include <mutex>

#include "rda_internal.h"
#include "rda_io.cuh"

namespace rda {
namespace {

constexpr int kTok = 32;          // tokens per pre-kernel CTA (one sequence)

__device__ __forceinline__ float sigmoid_f(float x) { return __frcp_rn(1.f + __expf(-x)); }
// Hardware tanh (PTX tanh.approx.f32, relative error about 2^-11).
__device__ __forceinline__ float tanh_hw(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// FAST: sigmoid(x) = (1 + tanh(x / 2)) / 2, so x sigmoid(x) = h + h tanh(h) with
// h = x / 2: three instructions.  Its error is far below bf16 rounding (2^-8),
// so bf16 outputs take it; fp32 outputs keep the correctly rounded form.
template <int ACT, bool FAST> __device__ __forceinline__ float act_t(float x) {
    if constexpr (ACT == RDA_ACT_SILU) {
        if constexpr (FAST) {
            const float h = 0.5f * x;
            return fmaf(h, tanh_hw(h), h);
        } else {
            return x * sigmoid_f(x);
        }
    } else if constexpr (ACT == RDA_ACT_SIGMOID) {
        if constexpr (FAST) return fmaf(0.5f, tanh_hw(0.5f * x), 0.5f);
        else return sigmoid_f(x);
    } else {
        return x;
    }
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// NC channels per lane (D = 32 NC).
template <typename Tio, int NC> struct Vec;
template <typename Tio> struct Vec<Tio, 4> {
    static __device__ __forceinline__ void ld(const Tio *p, float *x) {
        const float4 v = Io<Tio>::ld4(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    }
    static __device__ __forceinline__ void st(Tio *p, const float *x) {
        Io<Tio>::st4(p, make_float4(x[0], x[1], x[2], x[3]));
    }
};
template <typename Tio> struct Vec<Tio, 2> {
    static __device__ __forceinline__ void ld(const Tio *p, float *x) {
        x[0] = Io<Tio>::ld(p);
        x[1] = Io<Tio>::ld(p + 1);
    }
    static __device__ __forceinline__ void st(Tio *p, const float *x) {
        Io<Tio>::st(p, x[0]);
        Io<Tio>::st(p + 1, x[1]);
    }
};

struct PrepArgs {
    const void *raw[3];           // q, k, v projections [total, H, D]
    const float *w[3];            // conv taps [H*D, 3]
    const __nv_bfloat16 *win_in;  // [N, 3, C] or null
    __nv_bfloat16 *win_out;       // [N, 3, C] or null
    const float *beta_raw, *delta, *la_raw;
    const int32_t *cu_seqlens;
    int num_seqs, seq_len, H, Dk, Dv, C;
    bool channel;
    int act;
    void *out[3];                 // q, k, v for the core
    float *beta, *gamma, *log_alpha;
};

// Pairs of channels as float2 (paired fp32 arithmetic, fma.rn.f32x2).
template <typename Tio, int NP> struct Pairs;
template <int NP> struct Pairs<__nv_bfloat16, NP> {
    static __device__ __forceinline__ void ld(const __nv_bfloat16 *p, float2 *x) {
        if constexpr (NP == 2) {
            const uint2 u = *reinterpret_cast<const uint2 *>(p);
            x[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
            x[1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        } else {
            const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
            x[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
        }
    }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, const float2 *x) {
        if constexpr (NP == 2) {
            __nv_bfloat162 a = __float22bfloat162_rn(x[0]), b = __float22bfloat162_rn(x[1]);
            *reinterpret_cast<uint2 *>(p) =
                make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
        } else {
            __nv_bfloat162 a = __float22bfloat162_rn(x[0]);
            *reinterpret_cast<__nv_bfloat162 *>(p) = a;
        }
    }
};
template <int NP> struct Pairs<float, NP> {
    static __device__ __forceinline__ void ld(const float *p, float2 *x) {
        if constexpr (NP == 2) {
            const float4 v = *reinterpret_cast<const float4 *>(p);
            x[0] = make_float2(v.x, v.y);
            x[1] = make_float2(v.z, v.w);
        } else {
            x[0] = *reinterpret_cast<const float2 *>(p);
        }
    }
    static __device__ __forceinline__ void st(float *p, const float2 *x) {
        if constexpr (NP == 2) *reinterpret_cast<float4 *>(p) = make_float4(x[0].x, x[0].y, x[1].x, x[1].y);
        else *reinterpret_cast<float2 *>(p) = x[0];
    }
};

template <int ACT, bool FAST> __device__ __forceinline__ float2 act2(float2 x) {
    if constexpr (ACT == RDA_ACT_SILU && FAST) {
        const float2 h = __fmul2_rn(make_float2(0.5f, 0.5f), x);
        return __ffma2_rn(h, make_float2(tanh_hw(h.x), tanh_hw(h.y)), h);
    } else {
        return make_float2(act_t<ACT, FAST>(x.x), act_t<ACT, FAST>(x.y));
    }
}

// One CTA per (head, 32-token tile of a sequence): the tile's raw q, k and v
// rows of this head, with the two rows before it (the conv's history), go to
// shared memory first, all as 16-byte asynchronous copies issued up front
// (~26 KiB per CTA for bf16 at D = 128, eight CTAs per SM, whose load and
// compute phases interleave), then three warps compute from there: warp i owns
// tensor i (q, k, v); a lane owns 2 NP channels of a token row.
constexpr int kRowsT = kTok + 2;      // tile rows in shared memory: positions p0 - 2 .. p0 + kTok - 1
constexpr int kPrepWarps = 3;
constexpr int kTokW = kTok;           // tokens per warp
constexpr int kUnroll = 4;            // tokens per step of a warp's loop (independent reductions)

template <typename Tio, int DK, int DV>
struct PrepSmem {
    static constexpr uint32_t Q = 0;
    static constexpr uint32_t K = Q + kRowsT * DK * sizeof(Tio);
    static constexpr uint32_t V = K + kRowsT * DK * sizeof(Tio);
    static constexpr uint32_t BYTES = V + kRowsT * DV * sizeof(Tio);
};

// Tile rows [r_lo, r_hi) of head h of one tensor [rows, H, D] (tile row r =
// tensor row base_row + r) into shared memory, 16 bytes per copy.
template <typename Tio, int D>
__device__ __forceinline__ void issue_rows(uint32_t dst, const Tio *raw, int H, int h, long base_row, int r_lo,
                                           int r_hi) {
    constexpr int CPR = D * (int)sizeof(Tio) / 16;         // copies per row
    const int n = (r_hi - r_lo) * CPR;
    for (int e = threadIdx.x; e < n; e += kPrepWarps * 32) {
        const int r = r_lo + e / CPR, c = e % CPR;
        cp_async16(dst + (uint32_t)(r * D * sizeof(Tio) + c * 16),
                   reinterpret_cast<const char *>(raw + ((size_t)(base_row + r) * H + h) * D) + c * 16);
    }
}

// One warp's tokens [i0, i1) of one tensor: y_t = act(w0 x_{t-2} + w1 x_{t-1} +
// w2 x_t) from the rows in shared memory (row i + 2 holds x at tile position i),
// L2-normalised over the head for q and k, stored to the core's input.
template <typename Tio, int NP, int ACT>
__device__ __forceinline__ void conv_rows(const Tio *rows, Tio *dst, size_t stride, const float *w, int ch0,
                                          int i0, int i1, int lane, bool norm) {
    constexpr int NC = 2 * NP;
    constexpr int D = 32 * NC;
    constexpr bool FAST = sizeof(Tio) == 2;
    float2 w0[NP], w1[NP], w2[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const float *wj = w + (size_t)(ch0 + 2 * j) * 3;
        w0[j] = make_float2(wj[0], wj[3]);
        w1[j] = make_float2(wj[1], wj[4]);
        w2[j] = make_float2(wj[2], wj[5]);
    }
    const Tio *src = rows + lane * NC;
    float2 xm2[NP], xm1[NP];
    Pairs<Tio, NP>::ld(src + (size_t)i0 * D, xm2);
    Pairs<Tio, NP>::ld(src + (size_t)(i0 + 1) * D, xm1);
#pragma unroll 1
    for (int i = i0; i < i1; i += kUnroll) {
        float2 x[kUnroll][NP], y[kUnroll][NP];
        float ss[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) Pairs<Tio, NP>::ld(src + (size_t)(i + u + 2) * D, x[u]);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                float2 t = __fmul2_rn(w2[j], x[u][j]);
                t = __ffma2_rn(w1[j], xm1[j], t);
                t = __ffma2_rn(w0[j], xm2[j], t);
                y[u][j] = act2<ACT, FAST>(t);
                s2 = __ffma2_rn(y[u][j], y[u][j], s2);
                xm2[j] = xm1[j];
                xm1[j] = x[u][j];
            }
            ss[u] = s2.x + s2.y;
        }
        if (norm) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const float r = rsqrtf(ss[u]);
#pragma unroll
                for (int j = 0; j < NP; ++j) y[u][j] = __fmul2_rn(y[u][j], make_float2(r, r));
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            if (i + u < i1) Pairs<Tio, NP>::st(dst + (size_t)(i + u) * stride + lane * NC, y[u]);
    }
}

// grid (H, tiles of the longest sequence, sequences): the CTAs of one tile of
// all heads run side by side and read whole token rows.
template <typename Tio, int DK, int DV, int ACT>
__global__ void __launch_bounds__(kPrepWarps * 32, sizeof(Tio) == 2 ? 8 : 4) prep_inputs_kernel(PrepArgs a) {
    using L = PrepSmem<Tio, DK, DV>;
    extern __shared__ __align__(16) uint8_t psm[];
    const int n = blockIdx.z, h = blockIdx.x, tile = blockIdx.y;
    long t0, len;
    if (a.cu_seqlens) {
        t0 = a.cu_seqlens[n];
        len = (long)a.cu_seqlens[n + 1] - t0;
    } else {
        t0 = (long)n * a.seq_len;
        len = a.seq_len;
    }
    const long p0 = (long)tile * kTok;
    if (p0 >= len && !(tile == 0 && len == 0)) return;       // uniform across the CTA
    const int pend = (int)min((long)kTok, len - p0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.H;
    const uint32_t sb = static_cast<uint32_t>(__cvta_generic_to_shared(psm));
    const long base_row = t0 + p0 - 2;                      // sequence row of tile row 0
    // ---- the tile's rows: history rows from the sequence, or (first tile) from the window
    const int r_lo = tile == 0 ? 2 : 0;
    issue_rows<Tio, DK>(sb + L::Q, static_cast<const Tio *>(a.raw[0]), H, h, base_row, r_lo, pend + 2);
    issue_rows<Tio, DK>(sb + L::K, static_cast<const Tio *>(a.raw[1]), H, h, base_row, r_lo, pend + 2);
    issue_rows<Tio, DV>(sb + L::V, static_cast<const Tio *>(a.raw[2]), H, h, base_row, r_lo, pend + 2);
    cp_async_commit();
    if (tile == 0) {
        // positions -2 and -1: rows 1 and 2 of the carried window (oldest first), or zeros
        constexpr int CQ = DK, CV = DV;
        for (int e = threadIdx.x; e < 2 * (2 * CQ + CV); e += kPrepWarps * 32) {
            const int r = e / (2 * CQ + CV), c = e % (2 * CQ + CV);
            const int ti = c < CQ ? 0 : (c < 2 * CQ ? 1 : 2);
            const int d = ti == 0 ? c : (ti == 1 ? c - CQ : c - 2 * CQ);
            const int D = ti == 2 ? DV : DK;
            const int coff = ti == 0 ? 0 : (ti == 1 ? H * DK : 2 * H * DK);
            float x = 0.f;
            if (a.win_in) x = __bfloat162float(a.win_in[((size_t)n * 3 + r + 1) * a.C + coff + h * D + d]);
            Tio *rowp = reinterpret_cast<Tio *>(psm + (ti == 0 ? L::Q : (ti == 1 ? L::K : L::V)));
            Io<Tio>::st(rowp + r * D + d, x);
        }
    }
    // ---- the gates of the tile's tokens (their loads overlap the copies in flight)
    for (int i = threadIdx.x; i < pend; i += blockDim.x) {
        const size_t row = (size_t)(t0 + p0 + i) * H + h;
        const float br = a.beta_raw[row];
        const float be = sigmoid_f(br);
        a.beta[row] = be;
        if (a.gamma) a.gamma[row] = __fdividef(sigmoid_f(br + a.delta[row]), be);
        if (!a.channel) a.log_alpha[row] = fminf(fmaxf(a.la_raw[row], -5.f), 0.f);
    }
    if (a.channel) {
        for (int i = threadIdx.x; i < pend * DK; i += blockDim.x) {
            const size_t e = ((size_t)(t0 + p0 + i / DK) * H + h) * DK + i % DK;
            a.log_alpha[e] = fminf(fmaxf(a.la_raw[e], -5.f), 0.f);
        }
    }
    cp_async_wait_all();
    __syncthreads();
    // ---- q, k, v of the tile
    const int ti = warp;
    const int i0 = 0, i1 = min(kTokW, pend);
    if (i0 < i1) {
        const size_t row0 = (size_t)(t0 + p0) * H + h;
        if (ti < 2) {
            const Tio *rows = reinterpret_cast<const Tio *>(psm + (ti == 0 ? L::Q : L::K));
            Tio *dst = static_cast<Tio *>(a.out[ti]) + row0 * DK;
            conv_rows<Tio, DK / 64, ACT>(rows, dst, (size_t)H * DK, a.w[ti], h * DK + lane * (DK / 32), i0, i1,
                                         lane, true);
        } else {
            const Tio *rows = reinterpret_cast<const Tio *>(psm + L::V);
            Tio *dst = static_cast<Tio *>(a.out[2]) + row0 * DV;
            conv_rows<Tio, DV / 64, ACT>(rows, dst, (size_t)H * DV, a.w[2], h * DV + lane * (DV / 32), i0, i1,
                                         lane, false);
        }
    }
    // ---- the new window: the last three raw inputs of the sequence (shifting the
    // old window for sequences shorter than three); written by the first tile only,
    // after its own reads of the old window (the barrier above)
    if (tile == 0 && a.win_out) {
        const int CH = 2 * DK + DV;
        for (int e = threadIdx.x; e < 3 * CH; e += blockDim.x) {
            const int r = e / CH, c = e % CH;
            const int ti2 = c < DK ? 0 : (c < 2 * DK ? 1 : 2);
            const int d = ti2 == 0 ? c : (ti2 == 1 ? c - DK : c - 2 * DK);
            const int D = ti2 == 2 ? DV : DK;
            const int coff = ti2 == 0 ? 0 : (ti2 == 1 ? H * DK : 2 * H * DK);
            const long p = len - 3 + r;
            float x;
            if (p >= 0) {
                x = Io<Tio>::ld(static_cast<const Tio *>(a.raw[ti2]) + ((size_t)(t0 + p) * H + h) * D + d);
            } else {
                const long src = len + r;           // 0 .. 2: a row of the old window
                x = a.win_in ? __bfloat162float(a.win_in[((size_t)n * 3 + src) * a.C + coff + h * D + d]) : 0.f;
            }
            a.win_out[((size_t)n * 3 + r) * a.C + coff + h * D + d] = __float2bfloat16_rn(x);
        }
    }
}

struct PostArgs {
    const void *o, *g;
    const float *w;
    void *out;
    long rows;                    // tokens * H
    float eps;
    int act;
};

// kRows (token, head) rows of D = 32 NC values per warp, loads first
constexpr int kRows = 4;
template <typename Tio, int NC, int ACT>
__global__ void __launch_bounds__(256) output_gate_norm_kernel(PostArgs a) {
    const long row0 = ((long)blockIdx.x * 8 + (threadIdx.x >> 5)) * kRows;
    if (row0 >= a.rows) return;
    const int lane = threadIdx.x & 31;
    constexpr int D = 32 * NC;
    float o[kRows][4], g[kRows][4], w[4];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        if (row0 + r < a.rows) {
            const size_t off = (size_t)(row0 + r) * D + lane * NC;
            Vec<Tio, NC>::ld(static_cast<const Tio *>(a.o) + off, o[r]);
            Vec<Tio, NC>::ld(static_cast<const Tio *>(a.g) + off, g[r]);
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) o[r][c] = g[r][c] = 0.f;
        }
    }
#pragma unroll
    for (int c = 0; c < NC; ++c) w[c] = a.w[lane * NC + c];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        float ss = 0.f, y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < NC; ++c) ss = fmaf(o[r][c], o[r][c], ss);
        const float rn = rsqrtf(warp_sum(ss) / D + a.eps);
#pragma unroll
        for (int c = 0; c < NC; ++c) y[c] = o[r][c] * rn * w[c] * act_t<ACT, sizeof(Tio) == 2>(g[r][c]);
        if (row0 + r < a.rows) Vec<Tio, NC>::st(static_cast<Tio *>(a.out) + (size_t)(row0 + r) * D + lane * NC, y);
    }
}

template <typename T, int DK, int DV, int ACT>
cudaError_t launch_prep(dim3 grid, uint32_t smem, const PrepArgs &a, cudaStream_t s) {
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [smem] {
        attr = cudaFuncSetAttribute(prep_inputs_kernel<T, DK, DV, ACT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem);
    });
    if (attr != cudaSuccess) return attr;
    prep_inputs_kernel<T, DK, DV, ACT><<<grid, kPrepWarps * 32, smem, s>>>(a);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_prep_inputs(const PrepLaunch &l, cudaStream_t s) {
    PrepArgs a{};
    for (int i = 0; i < 3; ++i) {
        a.raw[i] = l.raw[i];
        a.w[i] = l.w[i];
        a.out[i] = l.out[i];
    }
    a.win_in = static_cast<const __nv_bfloat16 *>(l.win_in);
    a.win_out = static_cast<__nv_bfloat16 *>(l.win_out);
    a.beta_raw = l.beta_raw; a.delta = l.delta; a.la_raw = l.la_raw;
    a.cu_seqlens = l.cu_seqlens;
    a.num_seqs = l.num_seqs; a.seq_len = l.seq_len;
    a.H = l.H; a.Dk = l.Dk; a.Dv = l.Dv; a.C = l.H * (2 * l.Dk + l.Dv);
    a.channel = l.channel; a.act = l.act;
    a.beta = l.beta; a.gamma = l.gamma; a.log_alpha = l.log_alpha;
    const long tiles = (l.max_seqlen + kTok - 1) / kTok;
    const dim3 grid(l.H, (unsigned)(tiles > 0 ? tiles : 1), l.num_seqs);
    const bool f32 = l.dtype == RDA_F32;
    cudaError_t e = cudaSuccess;
#define RDA_PREP(T, DK, DV)                                                                     \
    do {                                                                                        \
        constexpr uint32_t smem = PrepSmem<T, DK, DV>::BYTES;                                   \
        if (l.act == RDA_ACT_SILU) e = launch_prep<T, DK, DV, RDA_ACT_SILU>(grid, smem, a, s);   \
        else e = launch_prep<T, DK, DV, RDA_ACT_NONE>(grid, smem, a, s);                         \
    } while (0)
    if (l.Dk == 128 && l.Dv == 128) { if (f32) RDA_PREP(float, 128, 128); else RDA_PREP(__nv_bfloat16, 128, 128); }
    else if (l.Dk == 128) { if (f32) RDA_PREP(float, 128, 64); else RDA_PREP(__nv_bfloat16, 128, 64); }
    else if (l.Dv == 128) { if (f32) RDA_PREP(float, 64, 128); else RDA_PREP(__nv_bfloat16, 64, 128); }
    else { if (f32) RDA_PREP(float, 64, 64); else RDA_PREP(__nv_bfloat16, 64, 64); }
#undef RDA_PREP
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_output_gate_norm(const void *o, const void *g, const float *w, void *out, long rows, int Dv,
                                    float eps, int act, rda_dtype_t dtype, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    PostArgs a{o, g, w, out, rows, eps, act};
    const unsigned grid = (unsigned)((rows + 8 * kRows - 1) / (8 * kRows));
#define RDA_POST(T, NC)                                                                          \
    do {                                                                                         \
        if (act == RDA_ACT_SIGMOID) output_gate_norm_kernel<T, NC, RDA_ACT_SIGMOID><<<grid, 256, 0, s>>>(a); \
        else if (act == RDA_ACT_SILU) output_gate_norm_kernel<T, NC, RDA_ACT_SILU><<<grid, 256, 0, s>>>(a);  \
        else output_gate_norm_kernel<T, NC, RDA_ACT_NONE><<<grid, 256, 0, s>>>(a);                            \
    } while (0)
    if (dtype == RDA_F32) {
        if (Dv == 128) RDA_POST(float, 4);
        else RDA_POST(float, 2);
    } else {
        if (Dv == 128) RDA_POST(__nv_bfloat16, 4);
        else RDA_POST(__nv_bfloat16, 2);
    }
#undef RDA_POST
    return cudaGetLastError();
}

}  // namespace rda
