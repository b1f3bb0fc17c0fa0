// Token-sequential fp32 prefill kernel.
//
// Evaluates the gated delta rule one token at a time (decay, error against the
// decayed state, write with strength beta, post-update read; article "Raon-1
// nano: half of a 3.1B model is a lookup table, and a 99M model keeps one too",
// section "The other 1.5B: a hybrid built to forget") with the state held in
// fp32 registers.  Each token uses the one-pass identity
//     a = S k,  b = S q,  e = gamma v - alpha a,
//     o = scale (alpha b + beta (k.q) e),  S <- alpha S + beta e k^T
// which equals decay-then-error-then-write exactly in real arithmetic.
//
// Value columns are independent under the rule (column j of S only meets v_j),
// so one CTA owns a 32-column slice of one (sequence, head); 8 warps own 4
// columns each and split the key rows across lanes; the two reductions over
// the key dimension are warp butterflies.
//
// With per-key-channel decay (log alpha [.., T, H, Dk]; key dim i of the state
// decays by alpha_i) the decayed state is S diag(alpha), so the same identity
// holds with the two reductions taken against alpha o k and alpha o q, the
// key-query product k.q unchanged, and each key row decayed by its own alpha:
//     e = gamma v - S (alpha o k),  o = scale (S (alpha o q) + beta (k.q) e),
//     S <- S diag(alpha) + beta e k^T
//
// This path serves fp32 inputs (held to fp32 accuracy), bf16 with Dk = 64, and
// every per-key-channel call.
#include "rda_internal.h"
#include "rda_io.cuh"

namespace rda {
namespace {

constexpr int kThreads = 256;
constexpr int kCols = 32;          // value columns per CTA
constexpr int kColsPerWarp = 4;
constexpr int kTile = 16;          // tokens staged in shared memory at a time

template <typename Tio, int DK, bool CH>
__global__ void __launch_bounds__(kThreads)
recurrent_kernel(PrefillArgs a) {
    constexpr int R = DK / 32;     // key rows per lane
    __shared__ float k_s[kTile][DK];
    __shared__ float q_s[kTile][DK];
    __shared__ float a_s[CH ? kTile : 1][DK];   // per-channel alpha
    __shared__ float v_s[kTile][kCols];
    __shared__ float o_s[kTile][kCols];
    __shared__ float g_s[kTile][3];    // alpha, beta, gamma

    const int slice = blockIdx.x, h = blockIdx.y;
    const int n = a.order ? a.order[blockIdx.z] : (int)blockIdx.z;
    long t0, len;
    if (a.cu_seqlens) {
        t0 = a.cu_seqlens[n];
        len = (long)a.cu_seqlens[n + 1] - t0;
    } else {
        t0 = (long)n * a.T;
        len = a.T;
    }
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int j0 = slice * kCols;
    const int jw = warp * kColsPerWarp;
    const int H = a.H, Dv = a.Dv;
    const Tio *q = static_cast<const Tio *>(a.q);
    const Tio *k = static_cast<const Tio *>(a.k);
    const Tio *v = static_cast<const Tio *>(a.v);
    Tio *out = static_cast<Tio *>(a.out);

    // S[r][c] = state element (key row lane + 32 r, value column j0 + jw + c)
    float S[R][4];
    const size_t sbase = ((size_t)n * H + h) * DK * Dv;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (a.s0) x = *reinterpret_cast<const float4 *>(a.s0 + sbase + (size_t)(lane + 32 * r) * Dv + j0 + jw);
        S[r][0] = x.x; S[r][1] = x.y; S[r][2] = x.z; S[r][3] = x.w;
    }

    for (long tb = 0; tb < len; tb += kTile) {
        const int nt = (int)min((long)kTile, len - tb);
        if (a.ckpt) {
            // the state entering this tile, for the backward pass: [seq][H][tile][Dk][Dv]
            const long ntile = (len + kTile - 1) / kTile;
            float *ck = a.ckpt + (((size_t)n * H + h) * ntile + tb / kTile) * DK * Dv;
#pragma unroll
            for (int r = 0; r < R; ++r)
                *reinterpret_cast<float4 *>(ck + (size_t)(lane + 32 * r) * Dv + j0 + jw) =
                    make_float4(S[r][0], S[r][1], S[r][2], S[r][3]);
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < nt * DK; idx += kThreads) {
            const int tt = idx / DK, d = idx % DK;
            const size_t row = (size_t)(t0 + tb + tt) * H + h;
            k_s[tt][d] = Io<Tio>::ld(k + row * DK + d);
            q_s[tt][d] = Io<Tio>::ld(q + row * DK + d);
            if constexpr (CH) a_s[tt][d] = expf(a.log_alpha[row * DK + d]);
        }
        for (int idx = threadIdx.x; idx < nt * kCols; idx += kThreads) {
            const int tt = idx / kCols, c = idx % kCols;
            const size_t row = (size_t)(t0 + tb + tt) * H + h;
            v_s[tt][c] = Io<Tio>::ld(v + row * Dv + j0 + c);
        }
        if (threadIdx.x < nt) {
            const size_t row = (size_t)(t0 + tb + threadIdx.x) * H + h;
            g_s[threadIdx.x][0] = CH ? 1.f : expf(a.log_alpha[row]);
            g_s[threadIdx.x][1] = a.beta[row];
            g_s[threadIdx.x][2] = a.gamma ? a.gamma[row] : 1.f;
        }
        __syncthreads();

        for (int tt = 0; tt < nt; ++tt) {
            float kk[R], qq[R], ka[R], qa[R], ar[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                kk[r] = k_s[tt][lane + 32 * r];
                qq[r] = q_s[tt][lane + 32 * r];
                ar[r] = CH ? a_s[tt][lane + 32 * r] : 1.f;
                ka[r] = CH ? ar[r] * kk[r] : kk[r];
                qa[r] = CH ? ar[r] * qq[r] : qq[r];
            }
            float red[9];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float sa = 0.f, sb = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    sa = fmaf(S[r][c], ka[r], sa);
                    sb = fmaf(S[r][c], qa[r], sb);
                }
                red[c] = sa;
                red[4 + c] = sb;
            }
            float kq = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r) kq = fmaf(kk[r], qq[r], kq);
            red[8] = kq;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                for (int m = 0; m < 9; ++m) red[m] += __shfl_xor_sync(0xffffffffu, red[m], off);

            const float al = g_s[tt][0], be = g_s[tt][1], ga = g_s[tt][2];
            float o_mine = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float e = ga * v_s[tt][jw + c] - al * red[c];
                const float o = a.scale * (al * red[4 + c] + be * e * red[8]);
                if (lane == c) o_mine = o;
                const float bee = be * e;
#pragma unroll
                for (int r = 0; r < R; ++r) S[r][c] = fmaf(CH ? ar[r] : al, S[r][c], bee * kk[r]);
            }
            if (lane < 4) o_s[tt][jw + lane] = o_mine;
        }
        __syncthreads();
        if (out) {
            for (int idx = threadIdx.x; idx < nt * kCols; idx += kThreads) {
                const int tt = idx / kCols, c = idx % kCols;
                const size_t row = (size_t)(t0 + tb + tt) * H + h;
                Io<Tio>::st(out + row * Dv + j0 + c, o_s[tt][c]);
            }
        }
    }

    if (a.sf) {
#pragma unroll
        for (int r = 0; r < R; ++r)
            *reinterpret_cast<float4 *>(a.sf + sbase + (size_t)(lane + 32 * r) * Dv + j0 + jw) =
                make_float4(S[r][0], S[r][1], S[r][2], S[r][3]);
    }
}

template <typename Tio, bool CH>
cudaError_t launch_t(const PrefillArgs &a, cudaStream_t s) {
    dim3 grid(a.Dv / kCols, a.H, a.num_seqs);
    if (a.Dk == 128)
        recurrent_kernel<Tio, 128, CH><<<grid, kThreads, 0, s>>>(a);
    else
        recurrent_kernel<Tio, 64, CH><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_recurrent(const PrefillArgs &a, rda_dtype_t dtype, cudaStream_t s) {
    if (a.num_seqs == 0) return cudaSuccess;
    if (a.channel_decay)
        return dtype == RDA_F32 ? launch_t<float, true>(a, s) : launch_t<__nv_bfloat16, true>(a, s);
    return dtype == RDA_F32 ? launch_t<float, false>(a, s) : launch_t<__nv_bfloat16, false>(a, s);
}

}  // namespace rda
