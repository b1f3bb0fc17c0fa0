// Backward pass of the RDA core: the gradients of a loss
// L = <d_out, out> + <d_final_state, final_state> with respect to q, k, v,
// log alpha, beta, the write gate and the initial state, evaluated token by
// token in fp32.  The pages never discuss training; this is reverse-mode
// differentiation of the rule as the nano article's section "The other 1.5B: a
// hybrid built to forget" orders it (decay, error against the decayed state,
// write with strength beta, read).
//
// In the [Dk][Dv] storage (X = S^T), a forward token is
//   Xd = alpha X,   e_j = gamma v_j - sum_d Xd[d][j] k_d,
//   X  = Xd + beta k e^T,   o_j = scale sum_d X[d][j] q_d
// and its reverse, with dX the adjoint of the token's output state:
//   dX += scale q do^T;            dq_d += scale sum_j X[d][j] do_j
//   g_j = sum_d dX[d][j] k_d;      de = beta g;      d_beta += e . g
//   dk_d += beta sum_j dX[d][j] e_j - sum_j Xd[d][j] de_j
//   dv = gamma de;                 d_gamma += v . de
//   dXd = dX - k de^T;             d_log_alpha += <dXd, Xd>;   dX <- alpha dXd
//
// States are needed in reverse order.  The forward kernel stores the state
// entering every 16-token tile (checkpoints in the workspace); the backward
// kernel walks the tiles in reverse, recomputes the states entering the tile's
// 4-token sub-tiles from the checkpoint, then for each sub-tile (in reverse)
// recomputes its decayed states Xd and errors e in registers and applies the
// reverse steps.  Value columns are independent under the rule, so each CTA
// owns 32 of them (8 warps x 4 columns, lanes over the key rows) and the
// adjoint dX of its columns stays in registers.  Gradients that sum over value
// columns (dq, dk, the gate gradients) are summed over the CTA's warps with
// shared-memory atomics and over the CTAs of a head with global fp32 atomics
// into outputs the host clears first; dv and the initial state's gradient
// belong to one CTA each.
#include "rda_internal.h"
#include "rda_io.cuh"

namespace rda {
namespace {

constexpr int kThreads = 256;
constexpr int kCols = 32;          // value columns per CTA
constexpr int kTile = 16;          // tokens per checkpoint (the forward kernel's tile)
constexpr int kSub = 4;            // tokens per recomputed sub-tile

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

template <typename Tio, int DK>
__global__ void __launch_bounds__(kThreads, 1) backward_kernel(BackwardArgs a) {
    constexpr int R = DK / 32;     // key rows per lane
    __shared__ float k_s[kTile][DK];
    __shared__ float q_s[kTile][DK];
    __shared__ float v_s[kTile][kCols];
    __shared__ float do_s[kTile][kCols];
    __shared__ float g_s[kTile][3];            // alpha, beta, gamma
    __shared__ float dq_s[kTile][DK];          // per-token sums over this CTA's columns
    __shared__ float dk_s[kTile][DK];
    __shared__ float dsc_s[kTile][3];          // d log alpha, d beta, d gamma

    const int slice = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int j0 = slice * kCols, jw = warp * 4;
    const int H = a.H, Dv = a.Dv, T = a.T;
    const long t0 = (long)n * T;
    const int ntile = (T + kTile - 1) / kTile;
    const Tio *q = static_cast<const Tio *>(a.q);
    const Tio *k = static_cast<const Tio *>(a.k);
    const Tio *v = static_cast<const Tio *>(a.v);
    const Tio *dout = static_cast<const Tio *>(a.d_out);
    const size_t sbase = ((size_t)n * H + h) * DK * Dv;

    // adjoint of the final state
    float dX[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (a.d_sf) x = *reinterpret_cast<const float4 *>(a.d_sf + sbase + (size_t)(lane + 32 * r) * Dv + j0 + jw);
        dX[r][0] = x.x; dX[r][1] = x.y; dX[r][2] = x.z; dX[r][3] = x.w;
    }

    for (int tile = ntile - 1; tile >= 0; --tile) {
        const long tb = (long)tile * kTile;
        const int nt = (int)min((long)kTile, (long)T - tb);
        __syncthreads();
        for (int idx = threadIdx.x; idx < kTile * DK; idx += kThreads) {
            const int tt = idx / DK, d = idx % DK;
            if (tt < nt) {
                const size_t row = (size_t)(t0 + tb + tt) * H + h;
                k_s[tt][d] = Io<Tio>::ld(k + row * DK + d);
                q_s[tt][d] = Io<Tio>::ld(q + row * DK + d);
            }
            dq_s[tt][d] = 0.f;
            dk_s[tt][d] = 0.f;
        }
        for (int idx = threadIdx.x; idx < nt * kCols; idx += kThreads) {
            const int tt = idx / kCols, c = idx % kCols;
            const size_t row = (size_t)(t0 + tb + tt) * H + h;
            v_s[tt][c] = Io<Tio>::ld(v + row * Dv + j0 + c);
            do_s[tt][c] = Io<Tio>::ld(dout + row * Dv + j0 + c);
        }
        if (threadIdx.x < kTile) {
            const int tt = threadIdx.x;
            if (tt < nt) {
                const size_t row = (size_t)(t0 + tb + tt) * H + h;
                g_s[tt][0] = expf(a.log_alpha[row]);
                g_s[tt][1] = a.beta[row];
                g_s[tt][2] = a.gamma ? a.gamma[row] : 1.f;
            }
            dsc_s[tt][0] = dsc_s[tt][1] = dsc_s[tt][2] = 0.f;
        }
        __syncthreads();

        // one forward token from X (in place); returns its decayed state and errors
        auto fwd = [&](float (&X)[R][4], int tt, float (&Xd)[R][4], float (&e)[4]) {
            const float al = g_s[tt][0], be = g_s[tt][1], ga = g_s[tt][2];
            float kk[R];
#pragma unroll
            for (int r = 0; r < R; ++r) kk[r] = k_s[tt][lane + 32 * r];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float p = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    Xd[r][c] = al * X[r][c];
                    p = fmaf(Xd[r][c], kk[r], p);
                }
                e[c] = ga * v_s[tt][jw + c] - warp_sum(p);
#pragma unroll
                for (int r = 0; r < R; ++r) X[r][c] = fmaf(be * kk[r], e[c], Xd[r][c]);
            }
        };

        // the states entering the tile's sub-tiles, from the checkpoint
        float st[kTile / kSub][R][4];
        {
            const float *ck = a.ckpt + (((size_t)n * H + h) * ntile + tile) * DK * Dv;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float4 x = *reinterpret_cast<const float4 *>(ck + (size_t)(lane + 32 * r) * Dv + j0 + jw);
                st[0][r][0] = x.x; st[0][r][1] = x.y; st[0][r][2] = x.z; st[0][r][3] = x.w;
            }
            float X[R][4], Xd[R][4], e[4];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) X[r][c] = st[0][r][c];
#pragma unroll
            for (int sb = 1; sb < kTile / kSub; ++sb) {
#pragma unroll
                for (int i = 0; i < kSub; ++i) {
                    const int tt = (sb - 1) * kSub + i;
                    if (tt < nt) fwd(X, tt, Xd, e);
                }
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int c = 0; c < 4; ++c) st[sb][r][c] = X[r][c];
            }
        }

#pragma unroll
        for (int sb = kTile / kSub - 1; sb >= 0; --sb) {
            if (sb * kSub >= nt) continue;
            // recompute the sub-tile: decayed states and errors of its tokens
            float Xds[kSub][R][4], es[kSub][4];
            {
                float X[R][4];
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int c = 0; c < 4; ++c) X[r][c] = st[sb][r][c];
#pragma unroll
                for (int i = 0; i < kSub; ++i)
                    if (sb * kSub + i < nt) fwd(X, sb * kSub + i, Xds[i], es[i]);
            }
            // reverse steps
#pragma unroll
            for (int i = kSub - 1; i >= 0; --i) {
                const int tt = sb * kSub + i;
                if (tt >= nt) continue;
                const float al = g_s[tt][0], be = g_s[tt][1], ga = g_s[tt][2];
                float kk[R], qq[R], dov[4];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    kk[r] = k_s[tt][lane + 32 * r];
                    qq[r] = q_s[tt][lane + 32 * r];
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) dov[c] = do_s[tt][jw + c];
                // dX += scale q do^T;  dq = scale X do (X the token's output state)
                float dqr[R];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    float acc = 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float x = fmaf(be * kk[r], es[i][c], Xds[i][r][c]);
                        acc = fmaf(x, dov[c], acc);
                        dX[r][c] = fmaf(a.scale * qq[r], dov[c], dX[r][c]);
                    }
                    dqr[r] = a.scale * acc;
                }
                // g = dX^T k;  de = beta g
                float de[4], dbeta = 0.f, dgam = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float p = 0.f;
#pragma unroll
                    for (int r = 0; r < R; ++r) p = fmaf(dX[r][c], kk[r], p);
                    const float gj = warp_sum(p);
                    de[c] = be * gj;
                    dbeta = fmaf(es[i][c], gj, dbeta);
                    dgam = fmaf(v_s[tt][jw + c], de[c], dgam);
                }
                // dk = beta dX e - Xd de;  dXd = dX - k de^T;  d log alpha = <dXd, Xd>
                float dkr[R], dla = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    float acc = 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        acc = fmaf(be * dX[r][c], es[i][c], acc);
                        acc = fmaf(-Xds[i][r][c], de[c], acc);
                        const float dxd = fmaf(-kk[r], de[c], dX[r][c]);
                        dla = fmaf(dxd, Xds[i][r][c], dla);
                        dX[r][c] = al * dxd;
                    }
                    dkr[r] = acc;
                }
                dla = warp_sum(dla);
                // sums over the CTA's columns
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    atomicAdd(&dq_s[tt][lane + 32 * r], dqr[r]);
                    atomicAdd(&dk_s[tt][lane + 32 * r], dkr[r]);
                }
                const size_t row = (size_t)(t0 + tb + tt) * H + h;
                if (lane < 4) a.dv[row * Dv + j0 + jw + lane] = ga * de[lane];
                if (lane == 0) {
                    atomicAdd(&dsc_s[tt][0], dla);
                    atomicAdd(&dsc_s[tt][1], dbeta);
                    atomicAdd(&dsc_s[tt][2], dgam);
                }
            }
        }
        __syncthreads();
        // the tile's sums over this CTA's columns into the outputs (other CTAs of
        // the head add theirs)
        for (int idx = threadIdx.x; idx < nt * DK; idx += kThreads) {
            const int tt = idx / DK, d = idx % DK;
            const size_t row = (size_t)(t0 + tb + tt) * H + h;
            atomicAdd(a.dq + row * DK + d, dq_s[tt][d]);
            atomicAdd(a.dk + row * DK + d, dk_s[tt][d]);
        }
        if (threadIdx.x < nt) {
            const int tt = threadIdx.x;
            const size_t row = (size_t)(t0 + tb + tt) * H + h;
            atomicAdd(a.d_log_alpha + row, dsc_s[tt][0]);
            atomicAdd(a.d_beta + row, dsc_s[tt][1]);
            if (a.d_gamma) atomicAdd(a.d_gamma + row, dsc_s[tt][2]);
        }
    }
    if (a.d_s0) {
#pragma unroll
        for (int r = 0; r < R; ++r)
            *reinterpret_cast<float4 *>(a.d_s0 + sbase + (size_t)(lane + 32 * r) * Dv + j0 + jw) =
                make_float4(dX[r][0], dX[r][1], dX[r][2], dX[r][3]);
    }
}

template <typename Tio>
cudaError_t launch_t(const BackwardArgs &a, cudaStream_t s) {
    const dim3 grid(a.Dv / kCols, a.H, a.B);
    if (a.Dk == 128) backward_kernel<Tio, 128><<<grid, kThreads, 0, s>>>(a);
    else backward_kernel<Tio, 64><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t backward_ckpt_bytes(int B, int T, int H, int Dk, int Dv) {
    const size_t ntile = ((size_t)T + kTile - 1) / kTile;
    return (size_t)B * H * ntile * Dk * Dv * sizeof(float);
}

cudaError_t launch_backward(const BackwardArgs &a, rda_dtype_t dtype, cudaStream_t s) {
    return dtype == RDA_F32 ? launch_t<float>(a, s) : launch_t<__nv_bfloat16>(a, s);
}

}  // namespace rda
