// Chunked tensor-core prefill for sm_100a (bf16 q/k/v, Dk = 128, fp32 state).
//
// The gated delta rule (article "Raon-1 nano: half of a 3.1B model is a lookup
// table, and a 99M model keeps one too", section "The other 1.5B: a hybrid
// built to forget": decay, error against the decayed state, write with
// strength beta, post-update read) is evaluated 64 tokens at a time.  For a
// chunk entered with state S (stored [Dk][Dv], i.e. S^T of the math state)
// and g_t = sum_{s<=t} log alpha_s inside the chunk:
//
//   A   = strictly_lower( diag(beta) (K K^T) o Gamma ),  Gamma_ts = e^{g_t - g_s}
//   T   = (I + A)^{-1}                                    (the UT transform)
//   W   = T diag(beta e^g) K,     U' = T diag(beta gamma) V
//   P   = (Q K^T) o Gamma  (causal, diagonal kept)
//   U   = U' - W S                                        (pseudo-values)
//   O   = scale (diag(e^g) Q S + P U)
//   S  <- e^{g_C} S + K^T diag(e^{g_C - g}) U
//
// which equals the token-by-token rule exactly in real arithmetic.
//
// Two kernels, both on the caller's stream:
//
//  1. prep (chunk-parallel; one CTA per (chunk, head) over every chunk of
//     every sequence at once).  Computes everything that does not depend on
//     the state: g, [Q;K] K^T on the tensor cores, P and A, the UT transform
//     (diagonal 16x16 blocks by forward substitution, off-diagonal blocks by
//     tf32 mma.sync), then W and U' on the tensor cores.  Writes W and P as
//     ready-to-use swizzled MMA operand images, U' and g, into the caller's
//     workspace (40.25 KiB per chunk and head at Dv = 128).
//
//  2. scan (sequential over the chunks of one (sequence, head, value slice)).
//     Carries the fp32 state in registers; per chunk issues -W S and Q S, then
//     K^T U~ and P U on the tensor cores and updates the state.  Value columns
//     are independent under the rule, so slicing is exact.
//
// Operands: bf16 in shared memory, fp32 accumulators in TMEM (tcgen05.mma),
// Q/K/V tiles by TMA, workspace images by bulk copies.  Every wait is
// bounded; on expiry the CTA records RDA_ERR_TIMEOUT in the caller's error
// word, stops issuing work and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "rda_internal.h"
#include "sm100_ptx.cuh"

namespace rda {
namespace {

using namespace ptx;

constexpr int kC = 64;            // chunk length
constexpr int kDK = 128;          // key dimension handled here
constexpr uint64_t kWaitNs = 4000000000ull;   // bounded waits: 4 s

// Per (chunk, head) prep image in the workspace.
constexpr uint32_t kImgW = 0;          // W, bf16 K-major SW128 image, 2 halves of 8 KiB
constexpr uint32_t kImgP = 16384;      // P, bf16 K-major SW128 image, 8 KiB
constexpr uint32_t kImgU = 24576;      // U', bf16, value slices of width NV, each [64][NV]
                                       // (then g: 64 fp32 after 64*Dv*2 bytes)

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded mbarrier wait.  try_wait suspends the thread in hardware until the
// phase completes or a short limit passes; the loop adds the overall bound.
__device__ __noinline__ bool wait_bar_slow(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                           int32_t *err) {
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 0;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 63) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kWaitNs) {
                *abort_flag = 1;
                atomicCAS(err, 0, (int32_t)RDA_ERR_TIMEOUT);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int32_t *err) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, abort_flag, err);
}

// Byte offset of 16-byte chunk `c` of row `row` in a tile whose rows are
// `rowbytes` long, in the canonical swizzle of that width (rows contiguous;
// address bits [4,7) XORed with bits [7,10)).
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t c, uint32_t rowbytes) {
    const uint32_t lin = row * rowbytes + c * 16;
    const uint32_t mask = rowbytes == 128 ? 7u : (rowbytes == 64 ? 3u : 1u);
    return lin ^ (((lin >> 7) & mask) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint4 pack8(const float *x) {
    return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
}
__device__ __forceinline__ void unpack8(uint4 u, float *x) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 hh = *reinterpret_cast<const __nv_bfloat162 *>(&w[i]);
        float2 f = __bfloat1622float2(hh);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

// ---------------------------------------------------------------------------
// UT transform.
// ---------------------------------------------------------------------------
constexpr int kLd = 68;   // fp32 row stride of the 64x64 work matrices in shared memory

__device__ __forceinline__ uint32_t f2tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// D += A(16x8, row) * B(8x8, col), tf32 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_tf32(float *d, const uint32_t *a, const uint32_t *b) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// T = (I + A)^{-1}, A strictly lower triangular 64x64 (fp32, stride kLd),
// by 16x16 blocks: diagonal blocks by forward substitution (fp32), then
//   T_ij = -T_ii * (sum_{m=j}^{i-1} A_im T_mj),  level by level in i - j,
// each product on the tensor cores (tf32 mma.sync, fp32 accumulate).
// Called by the 128 threads of one warpgroup (cw = 0..127).
__device__ __forceinline__ void ut_solve(const float *Af, float *Tf, float *Xs, int cw) {
    const int wq = cw >> 5, lane = cw & 31;
    if (cw < 64) {
        const int b = cw >> 4, j = cw & 15;
        const float *Ab = Af + (16 * b) * kLd + 16 * b;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int s = 0; s < i; ++s) {
                if (s & 1) acc1 = fmaf(Ab[i * kLd + s], x[s], acc1);
                else acc0 = fmaf(Ab[i * kLd + s], x[s], acc0);
            }
            x[i] = (i == j) ? 1.f : (i < j ? 0.f : -(acc0 + acc1));
        }
        float *Tb = Tf + (16 * b) * kLd + 16 * b;
#pragma unroll
        for (int i = 0; i < 16; ++i) Tb[i * kLd + j] = x[i];
    } else {
        // strictly upper 16x16 blocks are zero: 6 blocks x 16 rows x 4 float4
        for (int e = cw - 64; e < 6 * 64; e += 64) {
            const int blk = e >> 6, a = (e >> 2) & 15, c4 = (e & 3) * 4;
            const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            *reinterpret_cast<float4 *>(Tf + (16 * bi + a) * kLd + 16 * bj + c4) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    named_bar_sync(1, 128);
    const int g = lane >> 2, tg = lane & 3;
    float *xs = Xs + wq * 128;   // per-warp 16x8 scratch
#pragma unroll 1
    for (int L = 1; L <= 3; ++L) {
        const int units = 2 * (4 - L);
#pragma unroll 1
        for (int u = wq; u < units; u += 4) {
            const int j = u >> 1, nt = u & 1, i = j + L;
            // X (16x8) = A[16i.., 16j .. 16i) * T[16j .. 16i, 16j + 8nt ..]
            float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
            for (int k0 = 16 * j; k0 < 16 * i; k0 += 8) {
                uint32_t a[4], bb[2];
                const float *ar = Af + (16 * i + g) * kLd + k0 + tg;
                a[0] = f2tf32(ar[0]);
                a[1] = f2tf32(ar[8 * kLd]);
                a[2] = f2tf32(ar[4]);
                a[3] = f2tf32(ar[8 * kLd + 4]);
                const float *br = Tf + (k0 + tg) * kLd + 16 * j + 8 * nt + g;
                bb[0] = f2tf32(br[0]);
                bb[1] = f2tf32(br[4 * kLd]);
                mma_tf32(x, a, bb);
            }
            xs[g * 8 + 2 * tg] = x[0];
            xs[g * 8 + 2 * tg + 1] = x[1];
            xs[(g + 8) * 8 + 2 * tg] = x[2];
            xs[(g + 8) * 8 + 2 * tg + 1] = x[3];
            __syncwarp();
            // Z = T_ii X ; T_ij = -Z
            float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                uint32_t a[4], bb[2];
                const float *ar = Tf + (16 * i + g) * kLd + 16 * i + 8 * ks + tg;
                a[0] = f2tf32(ar[0]);
                a[1] = f2tf32(ar[8 * kLd]);
                a[2] = f2tf32(ar[4]);
                a[3] = f2tf32(ar[8 * kLd + 4]);
                bb[0] = f2tf32(xs[(8 * ks + tg) * 8 + g]);
                bb[1] = f2tf32(xs[(8 * ks + tg + 4) * 8 + g]);
                mma_tf32(z, a, bb);
            }
            float *tr = Tf + (16 * i + g) * kLd + 16 * j + 8 * nt + 2 * tg;
            tr[0] = -z[0];
            tr[1] = -z[1];
            tr[8 * kLd] = -z[2];
            tr[8 * kLd + 1] = -z[3];
            __syncwarp();
        }
        named_bar_sync(1, 128);
    }
}

// ---------------------------------------------------------------------------
// Kernel 1: prep.  One CTA per (global chunk, head).
// ---------------------------------------------------------------------------
constexpr int kPrepThreads = 192;     // warp 0 TMA, warp 1 MMA, warps 2..5 compute
constexpr uint32_t kPrepTmemCols = 256;
// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t PS_QK = 0;          // [Q;K]: half h at h*16384: rows 0..63 Q, 64..127 K
constexpr uint32_t PS_V = 32768;       // V [64 x 128]: 2 halves of 8 KiB (SW128)
constexpr uint32_t PS_P = 49152;       // P image (8 KiB)
constexpr uint32_t PS_AF = 57344;      // A fp32 [64][kLd]
constexpr uint32_t PS_TF = PS_AF + 64 * kLd * 4;
constexpr uint32_t PS_XS = PS_TF + 64 * kLd * 4;     // 4 x 16x8 fp32
constexpr uint32_t PS_G = PS_XS + 4 * 128 * 4;       // g, beta, beta*gamma, e^g, e^{ref-g}: 5 x 64 fp32
constexpr uint32_t PS_BAR = PS_G + 5 * 64 * 4;
constexpr uint32_t PS_TMEMPTR = PS_BAR + 4 * 8;
constexpr uint32_t PS_FLAGS = PS_TMEMPTR + 4;
constexpr uint32_t kPrepSmem = PS_FLAGS + 4 + 1024;
// regions reused once their first contents are consumed
constexpr uint32_t PS_TBG = PS_QK + 0;        // over Q half 0 (Q is read only by the first MMA)
constexpr uint32_t PS_TB = PS_QK + 16384;     // over Q half 1
constexpr uint32_t PS_WIMG = PS_V;            // W image over V (after W and U' are done)
constexpr uint32_t PS_UIMG = PS_AF;           // U' staging over A (after the solve)
// TMEM columns
constexpr uint32_t PT_QK = 0, PT_U = 0, PT_W = 128;
enum PrepBar { PB_FULL = 0, PB_QK, PB_TREADY, PB_WU };

struct PrepMaps {
    CUtensorMap q, k, v;
};

// Where chunk `gc` (global over all sequences) lives.
struct ChunkLoc {
    long t0;       // first token of the sequence
    long len;      // sequence length
    int c;         // chunk index within the sequence
};

__device__ __forceinline__ bool locate_chunk(const PrefillArgs &a, long gc, ChunkLoc &loc) {
    if (!a.cu_seqlens) {
        const long cps = (a.T + kC - 1) / kC;
        if (cps == 0) return false;
        const long n = gc / cps;
        if (n >= a.num_seqs) return false;
        loc.t0 = n * (long)a.T;
        loc.len = a.T;
        loc.c = (int)(gc - n * cps);
        return true;
    }
    const int32_t *cb = a.chunk_base;
    if (gc >= cb[a.num_seqs]) return false;
    int lo = 0, hi = a.num_seqs - 1;      // last n with cb[n] <= gc
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cb[mid] <= gc) lo = mid;
        else hi = mid - 1;
    }
    loc.t0 = a.cu_seqlens[lo];
    loc.len = (long)a.cu_seqlens[lo + 1] - loc.t0;
    loc.c = (int)(gc - cb[lo]);
    return true;
}

template <int NV>
__global__ void __launch_bounds__(kPrepThreads, 2)
prep_kernel(const __grid_constant__ PrepMaps maps, const PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    ChunkLoc loc;
    const long gc = blockIdx.x;
    if (!locate_chunk(a, gc, loc)) return;     // uniform across the CTA
    const int h = blockIdx.y;
    const int H = a.H, Dv = a.Dv;
    const int lenc = (int)min((long)kC, loc.len - (long)loc.c * kC);
    const long row0 = loc.t0 + (long)loc.c * kC;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + PS_BAR);
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(sm + PS_TMEMPTR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + PS_FLAGS);
    float *g_s = reinterpret_cast<float *>(sm + PS_G);
    float *b_s = g_s + 64, *bg_s = g_s + 128, *eg_s = g_s + 192, *eb_s = g_s + 256;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, kPrepTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    uint8_t *img = a.workspace_chunks + ((size_t)gc * H + h) * a.chunk_bytes;

    if (warp == 0) {
        if (lane == 0) {
            uint64_t *full = &bars[PB_FULL];
            mbar_arrive_expect_tx(full, 32768 + 64 * Dv * 2);
            const int r0 = (int)row0;
            tma_load_3d(sm + PS_QK + 0, &maps.q, full, 0, h, r0);
            tma_load_3d(sm + PS_QK + 8192, &maps.k, full, 0, h, r0);
            tma_load_3d(sm + PS_QK + 16384, &maps.q, full, 64, h, r0);
            tma_load_3d(sm + PS_QK + 24576, &maps.k, full, 64, h, r0);
            tma_load_3d(sm + PS_V, &maps.v, full, 0, h, r0);
            if (Dv == 128) tma_load_3d(sm + PS_V + 8192, &maps.v, full, 64, h, r0);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t qk = smem_u32(sm + PS_QK), vv = smem_u32(sm + PS_V);
            const uint32_t tbg = smem_u32(sm + PS_TBG), tb = smem_u32(sm + PS_TB);
            constexpr uint32_t ID_QK = idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t ID_W = idesc_bf16(64, 128, 0, 1);
            const uint32_t ID_U = Dv == 128 ? idesc_bf16(64, 128, 0, 1) : idesc_bf16(64, 64, 0, 1);
            bool ok = wait_bar(&bars[PB_FULL], 0, abort_flag, a.err);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_bf16(tmem + PT_QK, smem_desc(qk + off, 16, 1024, kSw128),
                             smem_desc(qk + off + 8192, 16, 1024, kSw128), ID_QK, kk > 0);
                }
                mma_commit(&bars[PB_QK]);
                ok = wait_bar(&bars[PB_TREADY], 0, abort_flag, a.err);
            }
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    // W = T diag(beta e^g) K ; U' = T diag(beta gamma) V  (B operands MN-major)
                    mma_bf16(tmem + PT_W, smem_desc(tbg + kk * 32, 16, 1024, kSw128),
                             smem_desc(qk + 8192 + kk * 2048, 16384, 1024, kSw128), ID_W, kk > 0);
                    mma_bf16(tmem + PT_U, smem_desc(tb + kk * 32, 16, 1024, kSw128),
                             smem_desc(vv + kk * 2048, 8192, 1024, kSw128), ID_U, kk > 0);
                }
                mma_commit(&bars[PB_WU]);
            }
        }
    } else {
        const int cw = threadIdx.x - 64;
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;              // TMEM lane
        const bool lo = lane < 16;
        const int m = 16 * q4 + lane;              // row of an M=64 accumulator (if lo)
        const uint32_t tq = tmem + ((uint32_t)(32 * q4) << 16);
        float *Af = reinterpret_cast<float *>(sm + PS_AF);
        float *Tf = reinterpret_cast<float *>(sm + PS_TF);
        float *Xs = reinterpret_cast<float *>(sm + PS_XS);

        // ---- gates: g = cumsum(log alpha) (masked past the end), beta, beta*gamma
        if (r < 64) {
            const bool valid = r < lenc;
            const size_t row = (size_t)(row0 + r) * H + h;
            float la = valid ? a.log_alpha[row] : 0.f;
            const float be = valid ? a.beta[row] : 0.f;
            const float ga = (valid && a.gamma) ? a.gamma[row] : 1.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, la, off);
                if (lane >= off) la += y;
            }
            g_s[r] = la;
            b_s[r] = be;
            bg_s[r] = be * ga;
        }
        named_bar_sync(1, 128);
        if (r >= 32 && r < 64) g_s[r] += g_s[31];
        named_bar_sync(1, 128);
        if (r < 64) {
            // e^{g_s}, and e^{ref - g_s} with ref = g at the first token of s's 16-block
            // (g is non-increasing, so 0 <= ref - g_s <= 80 and the factor stays finite)
            eg_s[r] = __expf(g_s[r]);
            eb_s[r] = __expf(g_s[r & ~15] - g_s[r]);
        }
        if (cw == 0 && !wait_bar(&bars[PB_QK], 0, abort_flag, a.err)) *abort_flag = 1;
        named_bar_sync(1, 128);
        if (!*abort_flag) {
            tc_fence_after();
            float x[64];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) tmem_ld16(tq + PT_QK + 16 * cc, x + 16 * cc);
            tmem_wait_ld();
            const int t = r & 63;
            const float gt = g_s[t];
            // e^{g_t - g_s} = e^{g_t - ref(s)} e^{ref(s) - g_s}, both factors bounded
            float ea[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) ea[b] = (16 * b <= t) ? __expf(gt - g_s[16 * b]) : 0.f;
            if (r < 64) {
                // P row t: (Q K^T)[t][s] e^{g_t - g_s}, s <= t  -> bf16 K-major SW128 image
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int s = 8 * cc + e;
                        y[e] = (s <= t) ? x[s] * ea[s >> 4] * eb_s[s] : 0.f;
                    }
                    *reinterpret_cast<uint4 *>(sm + PS_P + swz(t, cc, 128)) = pack8(y);
                }
            } else {
                // A row t: beta_t (K K^T)[t][s] e^{g_t - g_s}, s < t
                const float bt = b_s[t];
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    float y[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = 4 * c4 + e;
                        y[e] = (s < t) ? bt * x[s] * ea[s >> 4] * eb_s[s] : 0.f;
                    }
                    *reinterpret_cast<float4 *>(Af + t * kLd + 4 * c4) = make_float4(y[0], y[1], y[2], y[3]);
                }
            }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (!*abort_flag) {
            if (cw == 0) {
                bulk_store(img + kImgP, sm + PS_P, 8192);
                bulk_commit();
            }
            ut_solve(Af, Tf, Xs, cw);
            // T diag(beta e^g) and T diag(beta gamma) as bf16 K-major SW128 images
            {
                const int t = cw >> 1, half = cw & 1;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int s0 = 32 * half + 8 * cc;
                    const float4 t0 = *reinterpret_cast<const float4 *>(Tf + t * kLd + s0);
                    const float4 t1 = *reinterpret_cast<const float4 *>(Tf + t * kLd + s0 + 4);
                    const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                    float y1[8], y2[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        y1[e] = tv[e] * b_s[s0 + e] * eg_s[s0 + e];
                        y2[e] = tv[e] * bg_s[s0 + e];
                    }
                    *reinterpret_cast<uint4 *>(sm + PS_TBG + swz(t, 4 * half + cc, 128)) = pack8(y1);
                    *reinterpret_cast<uint4 *>(sm + PS_TB + swz(t, 4 * half + cc, 128)) = pack8(y2);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
        }
        named_bar_sync(1, 128);
        if (cw == 0 && !*abort_flag) {
            mbar_arrive(&bars[PB_TREADY]);
            if (!wait_bar(&bars[PB_WU], 0, abort_flag, a.err)) *abort_flag = 1;
        }
        named_bar_sync(1, 128);
        if (!*abort_flag) {
            tc_fence_after();
            // W rows -> bf16 K-major SW128 image (2 halves of 64 columns)
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float x[64];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) tmem_ld16(tq + PT_W + 64 * half + 16 * cc, x + 16 * cc);
                tmem_wait_ld();
                if (lo) {
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc)
                        *reinterpret_cast<uint4 *>(sm + PS_WIMG + half * 8192 + swz(m, cc, 128)) = pack8(x + 8 * cc);
                }
            }
            // U' rows -> bf16, value slices of width NV: slice s at s*64*NV*2, row m at m*NV*2
            for (int half = 0; half < Dv / 64; ++half) {
                float x[64];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) tmem_ld16(tq + PT_U + 64 * half + 16 * cc, x + 16 * cc);
                tmem_wait_ld();
                if (lo) {
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        const int col = 64 * half + 8 * cc;
                        const int sl = col / NV, cin = col % NV;
                        *reinterpret_cast<uint4 *>(sm + PS_UIMG + sl * (64 * NV * 2) + m * (NV * 2) + cin * 2) =
                            pack8(x + 8 * cc);
                    }
                }
            }
            fence_proxy_async_smem();
        }
        named_bar_sync(1, 128);
        if (cw == 0) {
            if (!*abort_flag) {
                bulk_store(img + kImgW, sm + PS_WIMG, 16384);
                bulk_store(img + kImgU, sm + PS_UIMG, 64 * Dv * 2);
                bulk_store(img + kImgU + 64 * Dv * 2, g_s, 256);
                bulk_commit();
            }
            bulk_wait_all();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kPrepTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Kernel 2: scan.  One CTA per (sequence, head, value slice of width NV).
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 192;     // warp 0 loads, warp 1 MMA, warps 2..5 compute
constexpr uint32_t kScanTmemCols = 256;
// per-stage shared memory (bytes): Q 16K | K 16K | W 16K | P 8K | U' <= 8K | g 256
constexpr uint32_t SS_Q = 0, SS_K = 16384, SS_W = 32768, SS_P = 49152, SS_U = 57344, SS_G = 65536;
constexpr uint32_t SS_STAGE = 66560;                  // 65 KiB (multiple of 1024)
constexpr uint32_t SC_S = 2 * SS_STAGE;               // state [128 x NV] bf16 MN-major (<= 16K)
constexpr uint32_t SC_U = SC_S + 16384;               // U  [64 x NV] (<= 8K)
constexpr uint32_t SC_UT = SC_U + 8192;               // U~ [64 x NV]
constexpr uint32_t SC_BAR = SC_UT + 8192;
constexpr int kScanBars = 8;
constexpr uint32_t SC_TMEMPTR = SC_BAR + kScanBars * 8;
constexpr uint32_t SC_FLAGS = SC_TMEMPTR + 4;
constexpr uint32_t kScanSmem = SC_FLAGS + 4 + 1024;
constexpr uint32_t ST_U = 0, ST_O1 = 64, ST_O2 = 128, ST_DS = 192;   // TMEM columns (NV <= 64)
enum ScanBar { SB_FULL0 = 0, SB_FULL1, SB_EMPTY0, SB_EMPTY1, SB_UDONE, SB_DSDONE, SB_SREADY, SB_UREADY };

struct ScanMaps {
    CUtensorMap q, k;
};

template <int NV>
__global__ void __launch_bounds__(kScanThreads, 1)
scan_kernel(const __grid_constant__ ScanMaps maps, const PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SC_BAR);
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(sm + SC_TMEMPTR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + SC_FLAGS);
    constexpr uint32_t VROW = NV * 2;
    constexpr uint32_t VSW = NV == 64 ? kSw128 : (NV == 32 ? kSw64 : kSw32);
    constexpr uint32_t VBYTES = 64 * VROW;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slice = blockIdx.x, h = blockIdx.y;
    const int n = a.order ? a.order[blockIdx.z] : (int)blockIdx.z;
    long t0, len, gc0;
    if (a.cu_seqlens) {
        t0 = a.cu_seqlens[n];
        len = (long)a.cu_seqlens[n + 1] - t0;
        gc0 = a.chunk_base[n];
    } else {
        t0 = (long)n * a.T;
        len = a.T;
        gc0 = (long)n * ((a.T + kC - 1) / kC);
    }
    const int nchunks = (int)((len + kC - 1) / kC);
    const int j0 = slice * NV;
    const int H = a.H, Dv = a.Dv;
    const size_t cb = a.chunk_bytes;

    if (threadIdx.x == 0) {
        // a stage is free again once its MMAs are done (commit) and the
        // compute warps have read its g and U' (arrive): two arrivals
        for (int i = 0; i < kScanBars; ++i) mbar_init(&bars[i], (i == SB_EMPTY0 || i == SB_EMPTY1) ? 2 : 1);
        *abort_flag = 0;
        fence_mbar_init();
        if (nchunks > 0) {
            prefetch_tensormap(&maps.q);
            prefetch_tensormap(&maps.k);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, kScanTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    if (warp == 0) {
        if (lane == 0) {
            for (int c = 0; c < nchunks; ++c) {
                const int st = c & 1;
                if (c >= 2 && !wait_bar(&bars[SB_EMPTY0 + st], ((c >> 1) - 1) & 1, abort_flag, a.err)) break;
                uint64_t *full = &bars[SB_FULL0 + st];
                uint8_t *stg = sm + st * SS_STAGE;
                const uint8_t *img = a.workspace_chunks + ((size_t)(gc0 + c) * H + h) * cb;
                mbar_arrive_expect_tx(full, 16384 * 3 + 8192 + VBYTES + 256);
                const int r0 = (int)(t0 + (long)c * kC);
                tma_load_3d(stg + SS_Q, &maps.q, full, 0, h, r0);
                tma_load_3d(stg + SS_Q + 8192, &maps.q, full, 64, h, r0);
                tma_load_3d(stg + SS_K, &maps.k, full, 0, h, r0);
                tma_load_3d(stg + SS_K + 8192, &maps.k, full, 64, h, r0);
                bulk_load(stg + SS_W, img + kImgW, 16384, full);
                bulk_load(stg + SS_P, img + kImgP, 8192, full);
                bulk_load(stg + SS_U, img + kImgU + (size_t)slice * VBYTES, VBYTES, full);
                bulk_load(stg + SS_G, img + kImgU + 64 * Dv * 2, 256, full);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t base = smem_u32(sm);
            const uint32_t ss = smem_u32(sm + SC_S), uu = smem_u32(sm + SC_U), ut = smem_u32(sm + SC_UT);
            constexpr uint32_t ID_NEG = idesc_bf16(64, NV, 0, 1, 1);
            constexpr uint32_t ID_O = idesc_bf16(64, NV, 0, 1);
            constexpr uint32_t ID_DS = idesc_bf16(128, NV, 1, 1);
            for (int c = 0; c < nchunks; ++c) {
                const int st = c & 1;
                const uint32_t ph = c & 1;
                const uint32_t stg = base + st * SS_STAGE;
                if (!wait_bar(&bars[SB_FULL0 + st], (c >> 1) & 1, abort_flag, a.err)) break;
                if (!wait_bar(&bars[SB_SREADY], ph, abort_flag, a.err)) break;
                tc_fence_after();
                // U = -W S (U' is added by the compute warps) ; O1 = Q S
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bs = smem_desc(ss + kk * 16 * VROW, 128 * VROW, 8 * VROW, VSW);
                    const uint32_t off = (kk >> 2) * 8192 + (kk & 3) * 32;
                    mma_bf16(tmem + ST_U, smem_desc(stg + SS_W + off, 16, 1024, kSw128), bs, ID_NEG, kk > 0);
                    mma_bf16(tmem + ST_O1, smem_desc(stg + SS_Q + off, 16, 1024, kSw128), bs, ID_O, kk > 0);
                }
                mma_commit(&bars[SB_UDONE]);
                if (!wait_bar(&bars[SB_UREADY], ph, abort_flag, a.err)) break;
                tc_fence_after();
                // dS = K^T U~ (A = K tile, MN-major) ; O2 = P U
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    mma_bf16(tmem + ST_DS, smem_desc(stg + SS_K + kk * 2048, 8192, 1024, kSw128),
                             smem_desc(ut + kk * 16 * VROW, VBYTES, 8 * VROW, VSW), ID_DS, kk > 0);
                    mma_bf16(tmem + ST_O2, smem_desc(stg + SS_P + kk * 32, 16, 1024, kSw128),
                             smem_desc(uu + kk * 16 * VROW, VBYTES, 8 * VROW, VSW), ID_O, kk > 0);
                }
                mma_commit(&bars[SB_DSDONE]);
                mma_commit(&bars[SB_EMPTY0 + st]);
            }
        }
    } else {
        const int cw = threadIdx.x - 64;
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const bool lo = lane < 16;
        const int m = 16 * q4 + lane;
        const uint32_t tq = tmem + ((uint32_t)(32 * q4) << 16);
        const size_t sbase = ((size_t)n * H + h) * kDK * Dv + (size_t)r * Dv + j0;
        __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(a.out);

        float S[NV];
#pragma unroll
        for (int j = 0; j < NV; j += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (a.s0) x = *reinterpret_cast<const float4 *>(a.s0 + sbase + j);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
        for (int c = 0; c < nchunks; ++c) {
            const int st = c & 1;
            const uint32_t ph = c & 1;
            const int lenc = (int)min((long)kC, len - (long)c * kC);
            const uint8_t *stg = sm + st * SS_STAGE;
            const float *g_s = reinterpret_cast<const float *>(stg + SS_G);
            // state -> bf16 MN-major operand
#pragma unroll
            for (int cc = 0; cc < NV / 8; ++cc)
                *reinterpret_cast<uint4 *>(sm + SC_S + swz(r, cc, VROW)) = pack8(S + 8 * cc);
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (cw == 0) {
                mbar_arrive(&bars[SB_SREADY]);
                // the stage's loads landed before the MMA warp used it; wait for
                // them here too, since g and U' are read directly below
                if (!wait_bar(&bars[SB_FULL0 + st], (c >> 1) & 1, abort_flag, a.err) ||
                    !wait_bar(&bars[SB_UDONE], ph, abort_flag, a.err))
                    *abort_flag = 1;
            }
            named_bar_sync(1, 128);
            if (*abort_flag) break;
            tc_fence_after();
            const float gC = g_s[63];
            // U = U' - W S ; U~ = e^{g_C - g} U
            {
                float x[NV];
#pragma unroll
                for (int cc = 0; cc < NV / 16; ++cc) tmem_ld16(tq + ST_U + 16 * cc, x + 16 * cc);
                tmem_wait_ld();
                if (lo) {
                    const uint8_t *urow = stg + SS_U + m * VROW;
#pragma unroll
                    for (int cc = 0; cc < NV / 8; ++cc) {
                        float u[8];
                        unpack8(*reinterpret_cast<const uint4 *>(urow + 16 * cc), u);
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[8 * cc + e] += u[e];
                    }
                    const float dec = __expf(gC - g_s[m]);
#pragma unroll
                    for (int cc = 0; cc < NV / 8; ++cc) {
                        *reinterpret_cast<uint4 *>(sm + SC_U + swz(m, cc, VROW)) = pack8(x + 8 * cc);
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = x[8 * cc + e] * dec;
                        *reinterpret_cast<uint4 *>(sm + SC_UT + swz(m, cc, VROW)) = pack8(y);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, 128);
            if (cw == 0) {
                mbar_arrive(&bars[SB_UREADY]);
                if (!wait_bar(&bars[SB_DSDONE], ph, abort_flag, a.err)) *abort_flag = 1;
            }
            named_bar_sync(1, 128);
            if (*abort_flag) break;
            tc_fence_after();
            // S <- e^{g_C} S + K^T U~
            {
                const float eC = __expf(gC);
                float x[NV];
#pragma unroll
                for (int cc = 0; cc < NV / 16; ++cc) tmem_ld16(tq + ST_DS + 16 * cc, x + 16 * cc);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < NV; ++j) S[j] = fmaf(eC, S[j], x[j]);
            }
            // O = scale (e^{g} Q S + P U)
            {
                float o1[NV], o2[NV];
#pragma unroll
                for (int cc = 0; cc < NV / 16; ++cc) {
                    tmem_ld16(tq + ST_O1 + 16 * cc, o1 + 16 * cc);
                    tmem_ld16(tq + ST_O2 + 16 * cc, o2 + 16 * cc);
                }
                tmem_wait_ld();
                if (lo && m < lenc) {
                    const float eg = __expf(g_s[m]) * a.scale;
                    const float sc = a.scale;
                    __nv_bfloat16 *orow = out + ((size_t)(t0 + (long)c * kC + m) * H + h) * Dv + j0;
#pragma unroll
                    for (int cc = 0; cc < NV / 8; ++cc) {
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = fmaf(eg, o1[8 * cc + e], sc * o2[8 * cc + e]);
                        *reinterpret_cast<uint4 *>(orow + 8 * cc) = pack8(y);
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(1, 128);
            if (cw == 0) mbar_arrive(&bars[SB_EMPTY0 + st]);
        }
        if (a.sf && !*abort_flag) {
#pragma unroll
            for (int j = 0; j < NV; j += 4)
                *reinterpret_cast<float4 *>(a.sf + sbase + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kScanTmemCols);
    }
}

// Exclusive prefix sum of ceil(len_n / 64) over packed sequences (one CTA).
__global__ void __launch_bounds__(1024) chunk_base_kernel(const int32_t *cu_seqlens, int num_seqs,
                                                          int32_t *chunk_base) {
    __shared__ int32_t wsum[32];
    __shared__ int32_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int base = 0; base < num_seqs; base += blockDim.x) {
        const int n = base + threadIdx.x;
        int32_t x = 0;
        if (n < num_seqs) x = (cu_seqlens[n + 1] - cu_seqlens[n] + kC - 1) / kC;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) wsum[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int32_t w = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, w, off);
                if (lane >= off) w += y;
            }
            wsum[lane] = w;
        }
        __syncthreads();
        const int32_t incl = x + (wid > 0 ? wsum[wid - 1] : 0) + carry;
        if (n < num_seqs) chunk_base[n + 1] = incl;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = incl;
        __syncthreads();
    }
    if (threadIdx.x == 0) chunk_base[0] = 0;
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool make_map(CUtensorMap *map, const void *base, int D, int H, long total_T, int box_d) {
    auto encode = get_encode();
    if (!encode) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)total_T};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {(cuuint32_t)box_d, 1u, (cuuint32_t)kC};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <typename K>
cudaError_t set_smem(K kernel, uint32_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

int choose_nv(long units, int Dv) {
    // The scan is latency-bound per chunk, so narrow slices cost little and
    // give more CTAs; widen them once the SMs are covered.
    if (units * (Dv / 64) >= 2 * 148) return 64;
    if (units * (Dv / 32) >= 148) return 32;
    return 16;
}

template <int NV>
cudaError_t launch_nv(const PrefillArgs &a, long chunks_grid, cudaStream_t s) {
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [] {
        attr = set_smem(prep_kernel<NV>, kPrepSmem);
        if (attr == cudaSuccess) attr = set_smem(scan_kernel<NV>, kScanSmem);
    });
    if (attr != cudaSuccess) return attr;
    PrepMaps pm;
    ScanMaps sm;
    std::memset(&pm, 0, sizeof(pm));
    std::memset(&sm, 0, sizeof(sm));
    if (a.total_T > 0) {
        if (!make_map(&pm.q, a.q, kDK, a.H, a.total_T, 64) || !make_map(&pm.k, a.k, kDK, a.H, a.total_T, 64) ||
            !make_map(&pm.v, a.v, a.Dv, a.H, a.total_T, 64))
            return cudaErrorInvalidValue;
        sm.q = pm.q;
        sm.k = pm.k;
    }
    if (chunks_grid > 0) {
        prep_kernel<NV><<<dim3((unsigned)chunks_grid, a.H, 1), kPrepThreads, kPrepSmem, s>>>(pm, a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    scan_kernel<NV><<<dim3(a.Dv / NV, a.H, a.num_seqs), kScanThreads, kScanSmem, s>>>(sm, a);
    return cudaGetLastError();
}

size_t image_bytes(int Dv) { return (size_t)kImgU + 64 * (size_t)Dv * 2 + 256; }

size_t header_bytes(int num_seqs) {
    size_t b = 4 * (size_t)(num_seqs + 1);
    return (b + 1023) / 1024 * 1024;
}

}  // namespace

bool chunked_supported(rda_dtype_t dtype, int Dk, int Dv) {
    return dtype == RDA_BF16 && Dk == kDK && (Dv == 64 || Dv == 128);
}

size_t chunked_workspace_bytes(long total_T, int T, int B, int H, int Dv, int num_seqs) {
    long chunks;
    if (num_seqs > 0) chunks = (total_T + kC - 1) / kC + num_seqs;     // packed: upper bound
    else chunks = (long)B * ((T + kC - 1) / kC);
    return header_bytes(num_seqs) + (size_t)chunks * H * image_bytes(Dv);
}

cudaError_t launch_chunked(const PrefillArgs &a0, void *scratch, cudaStream_t s) {
    PrefillArgs a = a0;
    uint8_t *ws = static_cast<uint8_t *>(scratch);
    a.workspace_chunks = ws + header_bytes(a.cu_seqlens ? a.num_seqs : 0);
    a.chunk_bytes = image_bytes(a.Dv);
    long chunks_grid;
    if (a.cu_seqlens) {
        int32_t *chunk_base = reinterpret_cast<int32_t *>(ws);
        a.chunk_base = chunk_base;
        chunk_base_kernel<<<1, 1024, 0, s>>>(a.cu_seqlens, a.num_seqs, chunk_base);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        chunks_grid = ((long)a.total_T + kC - 1) / kC + a.num_seqs;
    } else {
        a.chunk_base = nullptr;
        chunks_grid = (long)a.num_seqs * ((a.T + kC - 1) / kC);
    }
    if (a.total_T == 0) chunks_grid = 0;
    const long units = (long)a.num_seqs * a.H;
    switch (choose_nv(units, a.Dv)) {
        case 64: return launch_nv<64>(a, chunks_grid, s);
        case 32: return launch_nv<32>(a, chunks_grid, s);
        default: return launch_nv<16>(a, chunks_grid, s);
    }
}

}  // namespace rda
