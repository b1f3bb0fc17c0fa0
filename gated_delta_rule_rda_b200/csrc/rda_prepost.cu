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

#include "rda_internal.h"
#include "rda_io.cuh"

namespace rda {
namespace {

constexpr int kTok = 64;          // tokens per pre-kernel CTA (one sequence)
constexpr int kGrp = 2;           // tokens per step of the rolled token loop

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

// One tensor (q, k or v) of one head over one tile of a sequence, by one warp:
// 2 NP channels per lane; `norm`: L2-normalise each token over the head (q, k).
// q, k and v share this one code path (kept small for the instruction cache).
template <typename Tio, int NP, int ACT>
__device__ __forceinline__ void conv_tile(const Tio *raw, Tio *out, const float *w, const PrepArgs &a, int n, int h,
                                          int tile, long t0, long len, long p0, int pend, int coff, int lane,
                                          bool norm) {
    constexpr int NC = 2 * NP;
    constexpr int D = 32 * NC;
    constexpr bool FAST = sizeof(Tio) == 2;
    const int H = a.H;
    const int ch0 = h * D + lane * NC;                     // channel within the tensor
    const size_t stride = (size_t)H * D;                   // elements between tokens
    float2 w0[NP], w1[NP], w2[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const float *wj = w + (size_t)(ch0 + 2 * j) * 3;
        w0[j] = make_float2(wj[0], wj[3]);
        w1[j] = make_float2(wj[1], wj[4]);
        w2[j] = make_float2(wj[2], wj[5]);
    }
    const Tio *in = raw + (size_t)(t0 + p0) * stride + ch0;
    Tio *dst = out + (size_t)(t0 + p0) * stride + ch0;
    // window rows (positions -3, -2, -1 of the sequence), or zeros; tile 0 only
    float2 win[3][NP];
#pragma unroll
    for (int r = 0; r < 3; ++r)
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            win[r][j] = make_float2(0.f, 0.f);
            if (tile == 0 && a.win_in) {
                const __nv_bfloat16 *pw = a.win_in + ((size_t)n * 3 + r) * a.C + coff + ch0 + 2 * j;
                win[r][j] = make_float2(__bfloat162float(pw[0]), __bfloat162float(pw[1]));
            }
        }
    // the two inputs before the tile's first token
    float2 xm2[NP], xm1[NP];
    if (p0 >= 2) {
        Pairs<Tio, NP>::ld(in - 2 * stride, xm2);
        Pairs<Tio, NP>::ld(in - stride, xm1);
    } else {
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            xm2[j] = win[1][j];
            xm1[j] = win[2][j];
        }
    }
    auto load_grp = [&](int g0, float2 (&x)[kGrp][NP]) {
#pragma unroll
        for (int i = 0; i < kGrp; ++i) {
            if (g0 + i < pend) Pairs<Tio, NP>::ld(in + (size_t)(g0 + i) * stride, x[i]);
            else {
#pragma unroll
                for (int j = 0; j < NP; ++j) x[i][j] = make_float2(0.f, 0.f);
            }
        }
    };
    auto run_grp = [&](int g0, const float2 (&x)[kGrp][NP]) {
#pragma unroll
        for (int i = 0; i < kGrp; ++i) {
            float2 y[NP], ss2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                float2 t = __fmul2_rn(w2[j], x[i][j]);
                t = __ffma2_rn(w1[j], xm1[j], t);
                t = __ffma2_rn(w0[j], xm2[j], t);
                y[j] = act2<ACT, FAST>(t);
                ss2 = __ffma2_rn(y[j], y[j], ss2);
                xm2[j] = xm1[j];
                xm1[j] = x[i][j];
            }
            if (norm) {
                const float r = rsqrtf(warp_sum(ss2.x + ss2.y));
#pragma unroll
                for (int j = 0; j < NP; ++j) y[j] = __fmul2_rn(y[j], make_float2(r, r));
            }
            if (g0 + i < pend) Pairs<Tio, NP>::st(dst + (size_t)(g0 + i) * stride, y);
        }
    };
    // a rolled loop over pairs of token groups (a small body the instruction
    // cache keeps); each group's loads go out while the previous one computes
    float2 xa[kGrp][NP], xb[kGrp][NP];
    load_grp(0, xa);
#pragma unroll 1
    for (int g0 = 0; g0 < pend; g0 += 2 * kGrp) {
        load_grp(g0 + kGrp, xb);
        run_grp(g0, xa);
        if (g0 + kGrp >= pend) break;
        load_grp(g0 + 2 * kGrp, xa);
        run_grp(g0 + kGrp, xb);
    }
    // the new window: the last three raw inputs of the sequence (shifting the old
    // window for sequences shorter than three); written by the first tile only,
    // after its own reads of the old window
    if (tile == 0 && a.win_out) {
        const Tio *seq = raw + (size_t)t0 * stride + ch0;
#pragma unroll
        for (int r = 0; r < 3; ++r) {
            const long p = len - 3 + r;
            float2 v[NP];
            if (p >= 0) {
                Pairs<Tio, NP>::ld(seq + (size_t)p * stride, v);
            } else {
                const long src = len + r;           // 0 .. 2: a row of the old window
#pragma unroll
                for (int j = 0; j < NP; ++j) v[j] = src == 0 ? win[0][j] : (src == 1 ? win[1][j] : win[2][j]);
            }
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                __nv_bfloat16 *pw = a.win_out + ((size_t)n * 3 + r) * a.C + coff + ch0 + 2 * j;
                pw[0] = __float2bfloat16_rn(v[j].x);
                pw[1] = __float2bfloat16_rn(v[j].y);
            }
        }
    }
}

// grid (H, tiles of the longest sequence, sequences): the CTAs of one tile of
// all heads run side by side and read whole token rows; warps 0, 1, 2 own q,
// k, v.
template <typename Tio, int NCK, int NCV, int ACT>
__global__ void __launch_bounds__(96) prep_inputs_kernel(PrepArgs a) {
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
    const int coff = warp == 0 ? 0 : (warp == 1 ? H * a.Dk : 2 * H * a.Dk);
    const Tio *raw = static_cast<const Tio *>(warp == 0 ? a.raw[0] : (warp == 1 ? a.raw[1] : a.raw[2]));
    Tio *out = static_cast<Tio *>(warp == 0 ? a.out[0] : (warp == 1 ? a.out[1] : a.out[2]));
    const float *w = warp == 0 ? a.w[0] : (warp == 1 ? a.w[1] : a.w[2]);
    if (NCK == NCV || warp < 2)
        conv_tile<Tio, NCK / 2, ACT>(raw, out, w, a, n, h, tile, t0, len, p0, pend, coff, lane, warp < 2);
    else
        conv_tile<Tio, NCV / 2, ACT>(raw, out, w, a, n, h, tile, t0, len, p0, pend, coff, lane, false);

    // ---- gates of the tile's tokens
    for (int i = threadIdx.x; i < pend; i += blockDim.x) {
        const size_t row = (size_t)(t0 + p0 + i) * H + h;
        const float br = a.beta_raw[row];
        const float be = sigmoid_f(br);
        a.beta[row] = be;
        if (a.gamma) a.gamma[row] = __fdividef(sigmoid_f(br + a.delta[row]), be);
        if (!a.channel) a.log_alpha[row] = fminf(fmaxf(a.la_raw[row], -5.f), 0.f);
    }
    if (a.channel) {
        for (int i = threadIdx.x; i < pend * a.Dk; i += blockDim.x) {
            const size_t e = ((size_t)(t0 + p0 + i / a.Dk) * H + h) * a.Dk + i % a.Dk;
            a.log_alpha[e] = fminf(fmaxf(a.la_raw[e], -5.f), 0.f);
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
#define RDA_PREP(T, NK, NV)                                                         \
    do {                                                                            \
        if (l.act == RDA_ACT_SILU) prep_inputs_kernel<T, NK, NV, RDA_ACT_SILU><<<grid, 96, 0, s>>>(a); \
        else prep_inputs_kernel<T, NK, NV, RDA_ACT_NONE><<<grid, 96, 0, s>>>(a);   \
    } while (0)
    if (l.Dk == 128 && l.Dv == 128) { if (f32) RDA_PREP(float, 4, 4); else RDA_PREP(__nv_bfloat16, 4, 4); }
    else if (l.Dk == 128) { if (f32) RDA_PREP(float, 4, 2); else RDA_PREP(__nv_bfloat16, 4, 2); }
    else if (l.Dv == 128) { if (f32) RDA_PREP(float, 2, 4); else RDA_PREP(__nv_bfloat16, 2, 4); }
    else { if (f32) RDA_PREP(float, 2, 2); else RDA_PREP(__nv_bfloat16, 2, 2); }
#undef RDA_PREP
    return cudaGetLastError();
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
