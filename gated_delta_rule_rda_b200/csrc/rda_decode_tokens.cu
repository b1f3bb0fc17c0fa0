// Multi-token decode: T (1..8) new tokens per sequence in one pass over the
// state, as a speculative-decoding verifier needs (the model card
// "KRAFTON/Raon-1-nano-gguf", section "Model: KRAFTON/Raon-1-nano-gguf", runs
// multi-token prediction with drafts per step; the blog post on Raon-1 mini,
// section "Bạn có thể chạy gì trong tuần này", quotes a draft model at block
// size 8).  The result is that of T successive decode steps.
//
// Per value column j the state row s (key dim) after t tokens stays in the
// span of the old row and the new keys:
//     s_t = c_t s_0 + sum_{i<=t} w_i k_i,      c_t = alpha_1 ... alpha_t
// so the step needs, per column, only the 2T reductions a_t = s_0 . k_t and
// b_t = s_0 . q_t over the old state, plus the token Gram values k_i . k_t and
// k_i . q_t (shared by every column).  Then, token by token (scalar work):
//     p   = c_{t-1} a_t + sum_{i<t} w_i (k_i . k_t)       (= s_{t-1} . k_t)
//     e_t = gamma_t v_t - alpha_t p
//     w_i <- alpha_t w_i (i < t),  w_t = beta_t e_t,  c_t = alpha_t c_{t-1}
//     o_t = scale (c_t b_t + sum_{i<=t} w_i (k_i . q_t))
// and the new state is written once: S_new = c_T S_old + sum_i w_i k_i^T.
// The state is read and written once whatever T is, so T tokens cost about
// the HBM time of one decode step.
#include "rda_internal.h"
#include "rda_io.cuh"

namespace rda {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxT = kMaxDecodeTokens;

template <typename Tio, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 2)
decode_tokens_kernel(DecodeArgs a) {
    constexpr int TPR = DV / 4;              // threads across one state row
    constexpr int RG = kThreads / TPR;       // row groups
    constexpr int R = DK / RG;               // rows per thread
    extern __shared__ float4 red[];          // [2][T][RG][TPR]: partial a_t, then b_t
    __shared__ float k_s[kMaxT][DK];
    __shared__ float q_s[kMaxT][DK];
    __shared__ float v_s[kMaxT][DV];         // gamma_t v_t
    __shared__ __align__(16) float ab_s[2][kMaxT][DV];   // a_t = s_0 . k_t, b_t = s_0 . q_t per column
    __shared__ __align__(16) float w_s[kMaxT][DV];       // final coefficients w_i per column
    __shared__ float kk_s[kMaxT][kMaxT];     // [i][t] = k_i . k_t
    __shared__ float kq_s[kMaxT][kMaxT];     // [i][t] = k_i . q_t
    __shared__ float g_s[2][kMaxT];          // alpha, beta
    __shared__ float c_s;                    // c_T

    const int T = a.T, H = a.H;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int col4 = threadIdx.x % TPR;
    const int rg = threadIdx.x / TPR;
    float *st = a.state + (size_t)bh * DK * DV;
    auto tok = [&](int t) { return ((size_t)b * T + t) * H + h; };

    // Issue the state reads first; everything else overlaps their latency.
    float4 S[R];
#pragma unroll
    for (int r = 0; r < R; ++r)
        S[r] = __ldcs(reinterpret_cast<const float4 *>(st + (size_t)(rg + RG * r) * DV) + col4);

    for (int i = threadIdx.x; i < T * DK; i += kThreads) {
        const int t = i / DK, d = i % DK;
        k_s[t][d] = Io<Tio>::ld(static_cast<const Tio *>(a.k) + tok(t) * DK + d);
        q_s[t][d] = Io<Tio>::ld(static_cast<const Tio *>(a.q) + tok(t) * DK + d);
    }
    for (int i = threadIdx.x; i < T * DV; i += kThreads) {
        const int t = i / DV, j = i % DV;
        const float ga = a.gamma ? a.gamma[tok(t)] : 1.f;
        v_s[t][j] = ga * Io<Tio>::ld(static_cast<const Tio *>(a.v) + tok(t) * DV + j);
    }
    if (threadIdx.x < T) {
        const int t = threadIdx.x;
        g_s[0][t] = expf(a.log_alpha[tok(t)]);
        g_s[1][t] = a.beta[tok(t)];
    }
    __syncthreads();

    // token Gram values: 2 T^2 dot products over the key dim, one per warp at a time
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int p = warp; p < 2 * T * T; p += kThreads / 32) {
        const int which = p / (T * T), i = (p % (T * T)) / T, t = p % T;
        const float *x = which ? q_s[t] : k_s[t];
        float acc = 0.f;
        for (int d = lane; d < DK; d += 32) acc = fmaf(k_s[i][d], x[d], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) (which ? kq_s : kk_s)[i][t] = acc;
    }

    // partial products of the old state with every new key and query (paired
    // fp32 FMAs: two value columns per instruction)
    for (int t = 0; t < T; ++t) {
        float2 pa0 = make_float2(0.f, 0.f), pa1 = pa0, pb0 = pa0, pb1 = pa0;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float kr = k_s[t][rg + RG * r], qr = q_s[t][rg + RG * r];
            const float2 k2 = make_float2(kr, kr), q2 = make_float2(qr, qr);
            const float2 s0 = make_float2(S[r].x, S[r].y), s1 = make_float2(S[r].z, S[r].w);
            pa0 = __ffma2_rn(s0, k2, pa0); pa1 = __ffma2_rn(s1, k2, pa1);
            pb0 = __ffma2_rn(s0, q2, pb0); pb1 = __ffma2_rn(s1, q2, pb1);
        }
        red[(0 * T + t) * RG * TPR + rg * TPR + col4] = make_float4(pa0.x, pa0.y, pa1.x, pa1.y);
        red[(1 * T + t) * RG * TPR + rg * TPR + col4] = make_float4(pb0.x, pb0.y, pb1.x, pb1.y);
    }
    __syncthreads();

    // ... summed over the row groups: row group g finishes tokens g, g + RG, ...
    for (int t = rg; t < T; t += RG) {
        float4 at = make_float4(0.f, 0.f, 0.f, 0.f), bt = at;
#pragma unroll
        for (int g = 0; g < RG; ++g) {
            const float4 x = red[(0 * T + t) * RG * TPR + g * TPR + col4];
            const float4 y = red[(1 * T + t) * RG * TPR + g * TPR + col4];
            at.x += x.x; at.y += x.y; at.z += x.z; at.w += x.w;
            bt.x += y.x; bt.y += y.y; bt.z += y.z; bt.w += y.w;
        }
        *reinterpret_cast<float4 *>(&ab_s[0][t][4 * col4]) = at;
        *reinterpret_cast<float4 *>(&ab_s[1][t][4 * col4]) = bt;
    }
    __syncthreads();

    // the token recurrence, one value column per thread
    if (threadIdx.x < DV) {
        const int j = threadIdx.x;
        float c = 1.f;
        float w[kMaxT];
#pragma unroll
        for (int t = 0; t < kMaxT; ++t) {
            if (t >= T) break;
            float p = c * ab_s[0][t][j];
#pragma unroll
            for (int i = 0; i < t; ++i) p = fmaf(w[i], kk_s[i][t], p);
            const float al = g_s[0][t];
#pragma unroll
            for (int i = 0; i < t; ++i) w[i] *= al;
            w[t] = g_s[1][t] * (v_s[t][j] - al * p);
            c *= al;
            float o = c * ab_s[1][t][j];
#pragma unroll
            for (int i = 0; i <= t; ++i) o = fmaf(w[i], kq_s[i][t], o);
            Io<Tio>::st(static_cast<Tio *>(a.out) + tok(t) * DV + j, a.scale * o);
        }
#pragma unroll
        for (int t = 0; t < kMaxT; ++t) {
            if (t >= T) break;
            w_s[t][j] = w[t];
        }
        if (j == 0) c_s = c;
    }
    __syncthreads();

    // S_new = c_T S_old + sum_i w_i k_i^T, one write
    const float c = c_s;
    float4 w4[kMaxT];
#pragma unroll
    for (int i = 0; i < kMaxT; ++i)
        if (i < T) w4[i] = *reinterpret_cast<const float4 *>(&w_s[i][4 * col4]);
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int d = rg + RG * r;
        float2 s0 = make_float2(c * S[r].x, c * S[r].y), s1 = make_float2(c * S[r].z, c * S[r].w);
#pragma unroll
        for (int i = 0; i < kMaxT; ++i) {
            if (i >= T) break;
            const float kd = k_s[i][d];
            const float2 k2 = make_float2(kd, kd);
            s0 = __ffma2_rn(make_float2(w4[i].x, w4[i].y), k2, s0);
            s1 = __ffma2_rn(make_float2(w4[i].z, w4[i].w), k2, s1);
        }
        __stcs(reinterpret_cast<float4 *>(st + (size_t)d * DV) + col4, make_float4(s0.x, s0.y, s1.x, s1.y));
    }
}

template <typename Tio, int DK, int DV>
cudaError_t launch_shape(const DecodeArgs &a, cudaStream_t s) {
    constexpr int TPR = DV / 4, RG = kThreads / TPR;
    const size_t smem = 2 * (size_t)a.T * RG * TPR * sizeof(float4);
    static cudaError_t attr = cudaFuncSetAttribute(decode_tokens_kernel<Tio, DK, DV>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)(2 * kMaxT * RG * TPR * sizeof(float4)));
    if (attr != cudaSuccess) return attr;
    decode_tokens_kernel<Tio, DK, DV><<<(unsigned)(a.B * a.H), kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename Tio>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s) {
    if (a.Dk == 128 && a.Dv == 128) return launch_shape<Tio, 128, 128>(a, s);
    if (a.Dk == 128 && a.Dv == 64) return launch_shape<Tio, 128, 64>(a, s);
    if (a.Dk == 64 && a.Dv == 128) return launch_shape<Tio, 64, 128>(a, s);
    return launch_shape<Tio, 64, 64>(a, s);
}

}  // namespace

cudaError_t launch_decode_tokens(const DecodeArgs &a, rda_dtype_t dtype, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    return dtype == RDA_F32 ? launch_t<float>(a, s) : launch_t<__nv_bfloat16>(a, s);
}

}  // namespace rda
