// Fused one-pass decode step: one new token per sequence, state updated in place.
//
// The rule's T = 1 case (article "Raon-1 nano: half of a 3.1B model is a
// lookup table, and a 99M model keeps one too", section "The other 1.5B: a
// hybrid built to forget"), evaluated with a single read and a single write of
// the fp32 state:
//     a = S_old k,  b = S_old q               (two reductions over the key dim)
//     e = gamma v - alpha a
//     o = scale (alpha b + beta (k.q) e)
//     S_new = alpha S_old + beta e k^T
// The step is bound by HBM: 2 * Dk * Dv * 4 bytes of state per (sequence,
// head) against a few hundred bytes of token data.
//
// Per-key-channel decay (log alpha [B, H, Dk]): the decayed state is
// S_old diag(alpha) in the math orientation, i.e. row i of the [Dk][Dv]
// storage scales by alpha_i; with a = S_old (alpha o k), b = S_old (alpha o q):
//     e = gamma v - a,  o = scale (b + beta (k.q) e),  S_new = S_old diag(alpha) + beta e k^T.
//
// Layout of the work: one CTA per (sequence, head).  The state block
// [Dk][Dv] is row-major, so a warp reads whole rows with 16-byte loads
// (perfectly coalesced); each thread owns 4 value columns of DK/RG rows and
// keeps them in registers between the read and the write.  Partial sums over
// the thread's rows are combined across row groups through shared memory.
#include "rda_internal.h"
#include "rda_io.cuh"

namespace rda {
namespace {

constexpr int kThreads = 256;

template <typename Tio, int DK, int DV, bool CH>
__global__ void __launch_bounds__(kThreads, 2)
decode_kernel(DecodeArgs a) {
    constexpr int TPR = DV / 4;              // threads across one state row
    constexpr int RG = kThreads / TPR;       // row groups
    constexpr int R = DK / RG;               // rows per thread
    __shared__ float k_s[DK];
    __shared__ float q_s[DK];
    __shared__ float a_s[CH ? DK : 1];       // per-channel alpha
    __shared__ float4 red_a[RG][TPR];
    __shared__ float4 red_b[RG][TPR];
    __shared__ float kq_s;

    const int bh = blockIdx.x;
    const int col4 = threadIdx.x % TPR;
    const int rg = threadIdx.x / TPR;
    float *st = a.state + (size_t)bh * DK * DV;

    // Issue the state reads first; everything else overlaps their latency.
    float4 S[R];
#pragma unroll
    for (int r = 0; r < R; ++r)
        S[r] = __ldcs(reinterpret_cast<const float4 *>(st + (size_t)(rg + RG * r) * DV) + col4);

    const Tio *q = static_cast<const Tio *>(a.q) + (size_t)bh * DK;
    const Tio *k = static_cast<const Tio *>(a.k) + (size_t)bh * DK;
    for (int i = threadIdx.x; i < DK; i += kThreads) {
        k_s[i] = Io<Tio>::ld(k + i);
        q_s[i] = Io<Tio>::ld(q + i);
        if constexpr (CH) a_s[i] = expf(a.log_alpha[(size_t)bh * DK + i]);
    }
    const float4 vv = Io<Tio>::ld4(static_cast<const Tio *>(a.v) + (size_t)bh * DV + 4 * col4);
    const float al = CH ? 1.f : expf(a.log_alpha[bh]);
    const float be = a.beta[bh];
    const float ga = a.gamma ? a.gamma[bh] : 1.f;
    __syncthreads();

    if (threadIdx.x < 32) {
        float kq = 0.f;
        for (int i = threadIdx.x; i < DK; i += 32) kq = fmaf(k_s[i], q_s[i], kq);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (threadIdx.x == 0) kq_s = kq;
    }

    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float ar = CH ? a_s[rg + RG * r] : 1.f;
        const float kr = ar * k_s[rg + RG * r], qr = ar * q_s[rg + RG * r];
        pa.x = fmaf(S[r].x, kr, pa.x); pa.y = fmaf(S[r].y, kr, pa.y);
        pa.z = fmaf(S[r].z, kr, pa.z); pa.w = fmaf(S[r].w, kr, pa.w);
        pb.x = fmaf(S[r].x, qr, pb.x); pb.y = fmaf(S[r].y, qr, pb.y);
        pb.z = fmaf(S[r].z, qr, pb.z); pb.w = fmaf(S[r].w, qr, pb.w);
    }
    red_a[rg][col4] = pa;
    red_b[rg][col4] = pb;
    __syncthreads();

    float4 sa = make_float4(0.f, 0.f, 0.f, 0.f), sb = sa;
#pragma unroll
    for (int g = 0; g < RG; ++g) {
        const float4 x = red_a[g][col4], y = red_b[g][col4];
        sa.x += x.x; sa.y += x.y; sa.z += x.z; sa.w += x.w;
        sb.x += y.x; sb.y += y.y; sb.z += y.z; sb.w += y.w;
    }
    float4 e;
    e.x = ga * vv.x - al * sa.x;
    e.y = ga * vv.y - al * sa.y;
    e.z = ga * vv.z - al * sa.z;
    e.w = ga * vv.w - al * sa.w;

    if (rg == 0) {
        const float bkq = be * kq_s;
        float4 o;
        o.x = a.scale * (al * sb.x + bkq * e.x);
        o.y = a.scale * (al * sb.y + bkq * e.y);
        o.z = a.scale * (al * sb.z + bkq * e.z);
        o.w = a.scale * (al * sb.w + bkq * e.w);
        Io<Tio>::st4(static_cast<Tio *>(a.out) + (size_t)bh * DV + 4 * col4, o);
    }

    const float4 be4 = make_float4(be * e.x, be * e.y, be * e.z, be * e.w);
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float kr = k_s[rg + RG * r];
        const float ar = CH ? a_s[rg + RG * r] : al;
        float4 s = S[r];
        s.x = fmaf(ar, s.x, be4.x * kr);
        s.y = fmaf(ar, s.y, be4.y * kr);
        s.z = fmaf(ar, s.z, be4.z * kr);
        s.w = fmaf(ar, s.w, be4.w * kr);
        __stcs(reinterpret_cast<float4 *>(st + (size_t)(rg + RG * r) * DV) + col4, s);
    }
}

template <typename Tio, bool CH>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s) {
    const unsigned grid = (unsigned)(a.B * a.H);
    if (a.Dk == 128 && a.Dv == 128) decode_kernel<Tio, 128, 128, CH><<<grid, kThreads, 0, s>>>(a);
    else if (a.Dk == 128 && a.Dv == 64) decode_kernel<Tio, 128, 64, CH><<<grid, kThreads, 0, s>>>(a);
    else if (a.Dk == 64 && a.Dv == 128) decode_kernel<Tio, 64, 128, CH><<<grid, kThreads, 0, s>>>(a);
    else decode_kernel<Tio, 64, 64, CH><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, rda_dtype_t dtype, cudaStream_t s) {
    if (a.B == 0) return cudaSuccess;
    if (a.channel_decay)
        return dtype == RDA_F32 ? launch_t<float, true>(a, s) : launch_t<__nv_bfloat16, true>(a, s);
    return dtype == RDA_F32 ? launch_t<float, false>(a, s) : launch_t<__nv_bfloat16, false>(a, s);
}

}  // namespace rda
