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
// Two kernels on the caller's stream:
//
//  1. prep (chunk-parallel; one CTA per (chunk, head) over every chunk of
//     every sequence at once): everything the state chain and the outputs
//     need from a chunk.  g, K K^T and Q K^T on the tensor cores, A and P from
//     them, the UT transform (diagonal 16x16 blocks by forward substitution,
//     off-diagonal blocks by recursive doubling on tf32 mma.sync), then W and
//     U' on the tensor cores.  Writes -W and P as ready-to-use swizzled
//     operand images, U' in value slices and the decay factors.  Four CTAs per SM (55 KiB of shared memory, 128 TMEM
//     columns each): the Q, K, V, A and T tiles share three regions in turn.
//  2. scan (sequential over the chunks of one (sequence, head, value slice)).
//     Carries the fp32 state in registers; per chunk U = U' - W S and the
//     outputs O = scale (diag(e^g) (Q S) + P U) -- the two products with S
//     share its operand fragments; Q comes from the input by TMA -- then
//     S <- e^{g_C} S + K^T diag(e^{g_C - g}) U, on
//     register-fragment MMAs.  Value columns are independent under the rule,
//     so slicing is exact.
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

// Per (chunk, head) image in the workspace (bytes).
constexpr uint32_t kImgW = 0;          // -W, bf16 K-major SW128, 2 halves of 8 KiB (64 rows x 64 cols)
constexpr uint32_t kImgP = 16384;      // P, bf16 K-major SW128, 8 KiB
constexpr uint32_t kImgU = 24576;      // U', bf16, value slices of width NV, each [64][NV];
                                       // then e^{g_t} and e^{g_C - g_t}: 2 x 64 fp32
                                       // (per-key-channel decay: both 1, then e^{G_C} per key dim,
                                       // 128 fp32, then K~ = K o e^{G_C - G} and Q~ = Q o e^{G},
                                       // bf16 K-major SW128 like the K and Q tiles)
__host__ __device__ constexpr uint32_t img_decay(int Dv) { return kImgU + 64 * Dv * 2; }
__host__ __device__ constexpr uint32_t img_kt(int Dv) { return img_decay(Dv) + 1024; }
__host__ __device__ constexpr uint32_t img_qt(int Dv) { return img_kt(Dv) + 16384; }

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded mbarrier wait.  try_wait suspends the thread in hardware until the
// phase completes or a short limit passes; the loop adds the overall bound.
// Gives up when `stop` or `mine` is set, and sets `mine` when the bound runs
// out.  Threads that branch around named barriers on a flag pass it as both;
// a single-thread agent (TMA / MMA issue) passes its own `mine`, so that it
// never changes a flag such threads read.
__device__ __noinline__ bool wait_bar_slow(uint64_t *bar, uint32_t parity, volatile int *stop, volatile int *mine,
                                           int32_t *err, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 0;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 63) {
            if (*stop || *mine) return false;
            if (globaltimer() - t0 > limit_ns) {
                *mine = 1;
                atomicCAS(err, 0, (int32_t)RDA_ERR_TIMEOUT);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_bar2(uint64_t *bar, uint32_t parity, volatile int *stop, volatile int *mine,
                                          int32_t *err, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, stop, mine, err, limit_ns);
}
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *flag, int32_t *err,
                                         uint64_t limit_ns) {
    return wait_bar2(bar, parity, flag, flag, err, limit_ns);
}

// Bounded wait that ignores the abort flag: used only to let copies or MMAs
// already in flight land before a CTA that gave up exits.
__device__ __noinline__ void drain_bar(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > limit_ns) return;
}

// The dynamic shared memory rounded up to a 1024-byte boundary (what 128-byte
// swizzled tiles need).  Derived from the __shared__ array by pointer
// arithmetic, so that accesses through it stay shared-memory accesses.
__device__ __forceinline__ uint8_t *smem_align_1024(uint8_t *raw) {
    return raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
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

// T = (I + A)^{-1}, A strictly lower triangular 64x64 (fp32, stride kLd), by
// 16x16 blocks.  Diagonal blocks by forward substitution (fp32); then, by
// recursive doubling on [[X, 0], [Y, Z]]^-1 = [[X^-1, 0], [-Z^-1 Y X^-1, Z^-1]]:
//   the 16x16 blocks T_10 and T_32 (inside each 32-row half), then the 32x32
//   block T[32:64, 0:32] = -T[32:64, 32:64] A[32:64, 0:32] T[0:32, 0:32],
// each product on the tensor cores (tf32 mma.sync, fp32 accumulate).  The
// unused upper-right 32x32 block of A holds the intermediate product.
// Called by the 128 threads of one warpgroup (cw = 0..127).
__device__ __forceinline__ void ut_solve(float *Af, float *Tf, float *Xs, int cw) {
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
    // a tf32 A fragment (16x8) at (r0, k0) and B fragment (8x8) at (k0, c0) of
    // row-major fp32 matrices with stride kLd
    auto frag_a = [&](const float *m, int r0, int k0, uint32_t *a) {
        const float *ar = m + (r0 + g) * kLd + k0 + tg;
        a[0] = f2tf32(ar[0]);
        a[1] = f2tf32(ar[8 * kLd]);
        a[2] = f2tf32(ar[4]);
        a[3] = f2tf32(ar[8 * kLd + 4]);
    };
    auto frag_b = [&](const float *m, int k0, int c0, uint32_t *b) {
        const float *br = m + (k0 + tg) * kLd + c0 + g;
        b[0] = f2tf32(br[0]);
        b[1] = f2tf32(br[4 * kLd]);
    };
    {
        // T_{j+1,j}, j = 0 (warps 0, 1) or 2 (warps 2, 3), 8 columns per warp:
        // X = A_{j+1,j} T_jj, then -T_{j+1,j+1} X
        const int j = 2 * (wq >> 1), i = j + 1, c0 = 16 * j + 8 * (wq & 1);
        float *xs = Xs + wq * 128;       // per-warp 16x8 scratch
        float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k0 = 16 * j; k0 < 16 * i; k0 += 8) {
            uint32_t a[4], b[2];
            frag_a(Af, 16 * i, k0, a);
            frag_b(Tf, k0, c0, b);
            mma_tf32(x, a, b);
        }
        xs[g * 8 + 2 * tg] = x[0];
        xs[g * 8 + 2 * tg + 1] = x[1];
        xs[(g + 8) * 8 + 2 * tg] = x[2];
        xs[(g + 8) * 8 + 2 * tg + 1] = x[3];
        __syncwarp();
        float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t a[4], b[2];
            frag_a(Tf, 16 * i, 16 * i + 8 * ks, a);
            b[0] = f2tf32(xs[(8 * ks + tg) * 8 + g]);
            b[1] = f2tf32(xs[(8 * ks + tg + 4) * 8 + g]);
            mma_tf32(z, a, b);
        }
        float *tr = Tf + (16 * i + g) * kLd + c0 + 2 * tg;
        tr[0] = -z[0];
        tr[1] = -z[1];
        tr[8 * kLd] = -z[2];
        tr[8 * kLd + 1] = -z[3];
    }
    named_bar_sync(1, 128);
    // each warp one 16x16 quadrant (rows r0, columns c0) of the 32x32 products
    const int r0 = 16 * (wq >> 1), c0 = 16 * (wq & 1);
    {
        // Y = A[32:64, 0:32] T[0:32, 0:32] -> A[0:32, 32:64]  (T lower triangular:
        // rows above c0 contribute nothing to columns from c0)
        float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int k0 = 0; k0 < 32; k0 += 8) {
            if (k0 < c0) continue;
            uint32_t a[4];
            frag_a(Af, 32 + r0, k0, a);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                uint32_t b[2];
                frag_b(Tf, k0, c0 + 8 * nt, b);
                mma_tf32(y[nt], a, b);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float *yr = Af + (r0 + g) * kLd + 32 + c0 + 8 * nt + 2 * tg;
            yr[0] = y[nt][0];
            yr[1] = y[nt][1];
            yr[8 * kLd] = y[nt][2];
            yr[8 * kLd + 1] = y[nt][3];
        }
    }
    named_bar_sync(1, 128);
    {
        // T[32:64, 0:32] = -T[32:64, 32:64] Y  (T lower triangular: columns past
        // the quadrant's last row contribute nothing)
        float z[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int k0 = 0; k0 < 32; k0 += 8) {
            if (k0 >= r0 + 16) continue;
            uint32_t a[4];
            frag_a(Tf, 32 + r0, 32 + k0, a);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                uint32_t b[2];
                frag_b(Af, k0, 32 + c0 + 8 * nt, b);
                mma_tf32(z[nt], a, b);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float *tr = Tf + (32 + r0 + g) * kLd + c0 + 8 * nt + 2 * tg;
            tr[0] = -z[nt][0];
            tr[1] = -z[nt][1];
            tr[8 * kLd] = -z[nt][2];
            tr[8 * kLd + 1] = -z[nt][3];
        }
    }
    named_bar_sync(1, 128);
}

// ---------------------------------------------------------------------------
// Kernel 1: prep.  One CTA per (global chunk, head): everything the scan
// needs from a chunk -- g, A from K K^T, the UT transform T, then W and U' --
// and the chunk-local operand of the outputs, P = (Q K^T) o Gamma (causal,
// diagonal kept).
// Four CTAs share an SM (shared memory <= 55 KiB, 128 TMEM columns, <= 96
// registers): three regions are reused as the chunk's work moves along.
// ---------------------------------------------------------------------------
constexpr int kPrepThreads = 160;     // warp 0: TMEM and the tile loads; warps 1..4 compute (one of
                                      // their threads issues the MMAs and the V load)
constexpr uint32_t kPrepTmemCols = 128;
// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t PS_K = 0;           // K [64 x 128]: halves of 8 KiB (SW128); later the -W image
constexpr uint32_t PS_AF = 16384;      // A fp32 [64][kLd]; after the solve V [64 x Dv] (halves
                                       // of 8 KiB, SW128), after the U' MMA the U' slices
constexpr uint32_t PS_TF = PS_AF + 64 * kLd * 4;     // Q [64 x 128] (halves of 8 KiB, SW128) until the
                                                     // solve; T fp32 [64][kLd]; then the two T images
constexpr uint32_t PS_XS = PS_TF + 64 * kLd * 4;     // 4 x 16x8 fp32
constexpr uint32_t PS_G = PS_XS + 4 * 128 * 4;       // g, beta, beta*gamma, e^{ref-g}, e^g, e^{g_C-g}: 6 x 64 fp32,
                                                     // then (per-channel decay) e^{G_C} per key dim: 128 fp32
constexpr uint32_t PS_BAR = PS_G + 8 * 64 * 4;
constexpr uint32_t PS_TMEMPTR = PS_BAR + 10 * 8;
constexpr uint32_t PS_FLAGS = PS_TMEMPTR + 4;
constexpr uint32_t kPrepSmem = PS_FLAGS + 8 + 1024;   // flags: compute threads', TMA / MMA thread's
constexpr uint32_t PS_V = PS_AF;              // V, over A (loaded after the solve)
constexpr uint32_t PS_Q = PS_TF;              // Q, where T goes later
constexpr uint32_t PS_TBG = PS_TF;            // T diag(beta e^g), over T
constexpr uint32_t PS_TB = PS_TF + 8192;      // T diag(beta gamma)
constexpr uint32_t PS_WIMG = PS_K;            // -W image, over K (after the W MMA)
constexpr uint32_t PS_UIMG = PS_V;            // U' slices, over V (after the U' MMA)
static_assert(PS_AF % 1024 == 0 && PS_TF % 1024 == 0, "SW128 tiles need 1024-byte alignment");
static_assert(4 * (kPrepSmem + 1024) <= 233472, "four prep CTAs per SM");
// per-key-channel decay: the cumulative log decay G[t][d] of the chunk, fp32 [64][kGld]
constexpr int kGld = 132;
constexpr uint32_t PS_GCH = (kPrepSmem - 1024 + 15) / 16 * 16;
constexpr uint32_t kPrepSmemCh = PS_GCH + 64 * kGld * 4 + 1024;
static_assert(2 * (kPrepSmemCh + 1024) <= 233472, "two per-channel prep CTAs per SM");
// TMEM columns: K K^T and Q K^T side by side, then W, then U' (one at a time)
constexpr uint32_t PT_KK = 0, PT_QK = 64, PT_W = 0, PT_U = 0;
enum PrepBar { PB_FULL = 0, PB_VFULL, PB_KK, PB_QK, PB_W, PB_U, PB_DRAIN, kPrepBars };
static_assert(kPrepBars <= 10, "barrier area");

struct PrepMaps {
    CUtensorMap q, k, v;
};

// Which chunk a chunk-parallel CTA handles: `idx` enumerates every chunk of
// every sequence in order.
struct ChunkLoc {
    long t0;       // first token of the sequence
    long len;      // sequence length
    int c;         // chunk index within the sequence
    long gc;       // global chunk index: where its images live in the workspace
};

__device__ __forceinline__ bool locate_chunk(const PrefillArgs &a, long idx, ChunkLoc &loc) {
    loc.gc = idx;
    if (!a.cu_seqlens) {
        const long cps = (a.T + kC - 1) / kC;
        if (cps == 0) return false;
        const long n = idx / cps;
        if (n >= a.num_seqs) return false;
        loc.t0 = n * (long)a.T;
        loc.len = a.T;
        loc.c = (int)(idx - n * cps);
        return true;
    }
    const int32_t *cb = a.chunk_base;
    if (idx >= cb[a.num_seqs]) return false;
    int lo = 0, hi = a.num_seqs - 1;      // last n with cb[n] <= idx
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cb[mid] <= idx) lo = mid;
        else hi = mid - 1;
    }
    loc.t0 = a.cu_seqlens[lo];
    loc.len = (long)a.cu_seqlens[lo + 1] - loc.t0;
    loc.c = (int)(idx - cb[lo]);
    return true;
}

// Row r's gates (r < 64; zero decay and strength past the chunk's end).
struct RowGates {
    float la, be, ga;
};
__device__ __forceinline__ RowGates load_gates(const PrefillArgs &a, long row0, int lenc, int h, int r) {
    RowGates x{0.f, 0.f, 1.f};
    if (r < 64 && r < lenc) {
        const size_t row = (size_t)(row0 + r) * a.H + h;
        if (!a.channel_decay) x.la = a.log_alpha[row];
        x.be = a.beta[row];
        if (a.gamma) x.ga = a.gamma[row];
    }
    return x;
}
// Gates of one chunk, by the 128 compute threads (r = 0..127), from the rows'
// loaded gates: g = cumsum of log alpha (masked past the end), beta,
// beta*gamma and the decay factors.  Ends with a barrier of the compute threads.
__device__ __forceinline__ void chunk_gates(RowGates x, int r, int lane, float *g_s) {
    float *b_s = g_s + 64, *bg_s = g_s + 128, *eb_s = g_s + 192, *eg_s = g_s + 256, *ed_s = g_s + 320;
    if (r < 64) {
        float la = x.la;
        const float be = x.be, ga = x.ga;
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
        ed_s[r] = __expf(g_s[63] - g_s[r]);
    }
    named_bar_sync(1, 128);
}

// Two rows of a decayed, masked 64x64 Gram matrix from an M=64 TMEM accumulator
// (taddr at the warp's lane quarter), read with 16x256b loads so that all 32
// lanes hold data: thread l gets rows ta = 16 q + l/4 and ta + 8, and of each
// 8-column block kb the columns s = 8 kb + 2 (l%4) and s + 1, in
// v[4 kb .. 4 kb + 3] = (ta, s), (ta, s+1), (ta+8, s), (ta+8, s+1).
// On return v holds y = w_t X[t][s] e^{g_t - g_s} for s < t (strict) or s <= t,
// else 0; w_t = w_s[t], or 1 without w_s.
template <bool STRICT>
__device__ __forceinline__ void gram_rows(uint32_t taddr, int ta, int lane, const float *w_s, const float *g_s,
                                          float (&v)[32]) {
    const float *eb_s = g_s + 192;
    tmem_ld_16x256b_x4(taddr, v);
    tmem_ld_16x256b_x4(taddr + 32, v + 16);
    tmem_wait_ld();
    const int j2 = 2 * (lane & 3);
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int t = ta + 8 * rr;
        const float gt = g_s[t];
        const float w = w_s ? w_s[t] : 1.f;
        float ea[4];       // e^{g_t - g_s} = e^{g_t - ref(s)} e^{ref(s) - g_s}, both factors bounded
#pragma unroll
        for (int b = 0; b < 4; ++b) ea[b] = (16 * b <= t) ? w * __expf(gt - g_s[16 * b]) : 0.f;
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int s = 8 * kb + j2 + e;
                float &x = v[4 * kb + 2 * rr + e];
                x = (STRICT ? s < t : s <= t) ? x * ea[kb >> 1] * eb_s[s] : 0.f;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Per-key-channel decay: the decayed Grams.
//
// With one decay per key dim, the chunk's Gram entries are
//     X[t] . (K[s] o e^{G[t] - G[s]})   (X = K for A, Q for P),
// not a plain product times a mask.  Split the factor around a reference token
// r, e^{G[t] - G[r]} on the row operand and e^{G[r] - G[s]} on the column
// operand, and each 16 x 16 block is an ordinary product of scaled operands.
// The reference of every block of a row block is that row block's first token
// 16 rb: row factors <= 1; column factors <= 1 off the diagonal (s < r) and at
// most e^{15 x 5} on it (well inside the range of bf16 and fp32).  A factor
// that underflows belongs to an entry far below every other one in the row.
// So a row block's K and Q row operands serve all its blocks, and each column
// operand serves both the A and the P block of a pair.  The operands are scaled
// in fp32 and rounded to bf16 in the MMA fragments (mma.sync m16n8k16, fp32
// accumulation).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma16816_g(float *d, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Two consecutive key dims d, d + 1 of row t of a bf16 K-major SW128 tile
// (64-column halves of 8 KiB), scaled by e^{s (G[t][d] - G[ref][d])} (s = +-1),
// packed as a bf16 pair.
__device__ __forceinline__ uint32_t scaled_pair(const uint8_t *tile, const float *Gm, int t, int d, int ref,
                                                float sgn) {
    const uint32_t raw = *reinterpret_cast<const uint32_t *>(tile + (d >> 6) * 8192 + swz(t, (d & 63) >> 3, 128) +
                                                             (d & 7) * 2);
    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw));
    const float2 gt = *reinterpret_cast<const float2 *>(Gm + t * kGld + d);
    const float2 gr = *reinterpret_cast<const float2 *>(Gm + ref * kGld + d);
    return pack_bf16(x.x * __expf(sgn * (gt.x - gr.x)), x.y * __expf(sgn * (gt.y - gr.y)));
}
// Row block rb of the decayed Grams, by one warp: accK[cb] (A, before beta and
// the mask) and accQ[cb] (P, before the mask) for the column blocks cb <= rb,
// n-tiles of 8 columns, mma.sync accumulator layout.
__device__ __forceinline__ void gram_rowblock_ch(const uint8_t *kt, const uint8_t *qt, const float *Gm, int rb,
                                                 int lane, float (&accK)[4][2][4], float (&accQ)[4][2][4]) {
    const int g = lane >> 2, tg = lane & 3;
    const int t0 = 16 * rb + g, t1 = t0 + 8, ref = 16 * rb;
#pragma unroll 1
    for (int ks = 0; ks < 8; ++ks) {
        const int d = 16 * ks + 2 * tg;
        uint32_t ak[4], aq[4];
        ak[0] = scaled_pair(kt, Gm, t0, d, ref, 1.f);
        ak[1] = scaled_pair(kt, Gm, t1, d, ref, 1.f);
        ak[2] = scaled_pair(kt, Gm, t0, d + 8, ref, 1.f);
        ak[3] = scaled_pair(kt, Gm, t1, d + 8, ref, 1.f);
        aq[0] = scaled_pair(qt, Gm, t0, d, ref, 1.f);
        aq[1] = scaled_pair(qt, Gm, t1, d, ref, 1.f);
        aq[2] = scaled_pair(qt, Gm, t0, d + 8, ref, 1.f);
        aq[3] = scaled_pair(qt, Gm, t1, d + 8, ref, 1.f);
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            if (cb > rb) continue;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int sc = 16 * cb + 8 * nt + g;
                const uint32_t b0 = scaled_pair(kt, Gm, sc, d, ref, -1.f);
                const uint32_t b1 = scaled_pair(kt, Gm, sc, d + 8, ref, -1.f);
                mma16816_g(accK[cb][nt], ak, b0, b1);
                mma16816_g(accQ[cb][nt], aq, b0, b1);
            }
        }
    }
}

// The per-channel prep's work up to the UT solve, by the 128 compute threads
// (cw = 0..127; r = the thread's TMEM lane, the token whose gates it loaded):
// the cumulative log decay G[t][d] of every key dim, beta and beta*gamma; the
// decayed Grams A (strictly lower, rows times beta_t) into the fp32 work matrix
// and P (lower, diagonal kept) as its image; the images K~ = K o e^{G_C - G} and
// Q~ = Q o e^{G}; and K o e^{G} in place of the K tile (the B operand of W).
// The scalar decay factors of the image are set to 1 and e^{G_C} per key dim
// follows them.
__device__ __forceinline__ void prep_channel_front(const PrefillArgs &a, uint8_t *sm, float *g_s, RowGates gates,
                                                   int cw, int r, int lenc, long row0, int h, uint8_t *img,
                                                   uint64_t *bars, volatile int *abort_flag) {
    const int lane = cw & 31, wq = cw >> 5;
    float *b_s = g_s + 64, *bg_s = g_s + 128, *eg_s = g_s + 256, *ed_s = g_s + 320, *dc_s = g_s + 384;
    float *Gm = reinterpret_cast<float *>(sm + PS_GCH);
    const int H = a.H;
    {
        // key dim cw: G[t] = sum of log alpha over the chunk's tokens up to t (0 past the end)
        const float *la = a.log_alpha + ((size_t)row0 * H + h) * kDK + cw;
        const size_t step = (size_t)H * kDK;
        float x[64];
#pragma unroll
        for (int t = 0; t < 64; ++t) x[t] = t < lenc ? la[t * step] : 0.f;
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t < 64; ++t) {
            acc += x[t];
            Gm[t * kGld + cw] = acc;
        }
        dc_s[cw] = __expf(acc);
    }
    if (r < 64) {
        b_s[r] = gates.be;
        bg_s[r] = gates.be * gates.ga;
        eg_s[r] = 1.f;
        ed_s[r] = 1.f;
    }
    if (cw == 0 && !wait_bar(&bars[PB_FULL], 0, abort_flag, a.err, a.wait_ns)) *abort_flag = 1;
    named_bar_sync(1, 128);
    // only compute thread 0 writes the flag, and only before the barrier: uniform
    const bool go = !*abort_flag;
    // the tiles have landed (complete already); this wait makes the copies visible here
    if (go) wait_bar(&bars[PB_FULL], 0, abort_flag, a.err, a.wait_ns);
    float *Af = reinterpret_cast<float *>(sm + PS_AF);
    const uint8_t *kt = sm + PS_K, *qt = sm + PS_Q;
    const int g = lane >> 2, tg = lane & 3;
    if (go) {
        // warp wq owns row block 3 - wq: the largest first
        const int rb = 3 - wq;
        float accK[4][2][4], accQ[4][2][4];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) accK[cb][nt][i] = accQ[cb][nt][i] = 0.f;
        gram_rowblock_ch(kt, qt, Gm, rb, lane, accK, accQ);
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            if (cb > rb) continue;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int t = 16 * rb + g + 8 * hh, s0 = 16 * cb + 8 * nt + 2 * tg;
                    const float k0 = accK[cb][nt][2 * hh], k1 = accK[cb][nt][2 * hh + 1];
                    const float q0 = accQ[cb][nt][2 * hh], q1 = accQ[cb][nt][2 * hh + 1];
                    const float be = b_s[t];
                    *reinterpret_cast<float2 *>(Af + t * kLd + s0) =
                        make_float2(s0 < t ? be * k0 : 0.f, s0 + 1 < t ? be * k1 : 0.f);
                    *reinterpret_cast<uint32_t *>(img + kImgP + swz(t, s0 >> 3, 128) + (s0 & 7) * 2) =
                        pack_bf16(s0 <= t ? q0 : 0.f, s0 + 1 <= t ? q1 : 0.f);
                }
        }
    }
    // the blocks of P's image above the diagonal are zero (the scan multiplies by all 64 columns)
    for (int i = cw; go && i < 6 * 16 * 8; i += 128) {
        const int blk = i >> 7, t = (i >> 3) & 15, pr = i & 7;
        const int rb = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
        const int cb = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
        const int tt = 16 * rb + t, s0 = 16 * cb + 2 * pr;
        *reinterpret_cast<uint32_t *>(img + kImgP + swz(tt, s0 >> 3, 128) + (s0 & 7) * 2) = 0u;
    }
    named_bar_sync(1, 128);
    if (go) {
        // key dims dp, dp + 1 of rows 32 th .. 32 th + 31
        const int dp = 2 * (cw & 63), th = cw >> 6;
        const float2 gC = *reinterpret_cast<const float2 *>(Gm + 63 * kGld + dp);
        uint8_t *kimg = img + img_kt(a.Dv), *qimg = img + img_qt(a.Dv);
        for (int t = 32 * th; t < 32 * th + 32; ++t) {
            const uint32_t off = (dp >> 6) * 8192 + swz(t, (dp & 63) >> 3, 128) + (dp & 7) * 2;
            const float2 gt = *reinterpret_cast<const float2 *>(Gm + t * kGld + dp);
            const uint32_t kr = *reinterpret_cast<const uint32_t *>(sm + PS_K + off);
            const uint32_t qr = *reinterpret_cast<const uint32_t *>(sm + PS_Q + off);
            const float2 kx = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kr));
            const float2 qx = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&qr));
            const float e0 = __expf(gt.x), e1 = __expf(gt.y);
            *reinterpret_cast<uint32_t *>(kimg + off) =
                pack_bf16(kx.x * __expf(gC.x - gt.x), kx.y * __expf(gC.y - gt.y));
            *reinterpret_cast<uint32_t *>(qimg + off) = pack_bf16(qx.x * e0, qx.y * e1);
            *reinterpret_cast<uint32_t *>(sm + PS_K + off) = pack_bf16(kx.x * e0, kx.y * e1);
        }
    }
}

template <int NV, bool CH>
__global__ void __launch_bounds__(kPrepThreads, CH ? 2 : 4)
prep_kernel(const __grid_constant__ PrepMaps maps, const PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_align_1024(smem_raw);
    // the scan may launch (and run its prologue) once every prep CTA has started;
    // it waits for this grid's completion before it reads the workspace
    if (threadIdx.x == 0) pdl_launch_dependents();
    ChunkLoc loc;
    if (!locate_chunk(a, blockIdx.x, loc)) return;     // uniform across the CTA
    const long gc = loc.gc;
    const int h = blockIdx.y;
    const int H = a.H, Dv = a.Dv;
    const int lenc = (int)min((long)kC, loc.len - (long)loc.c * kC);
    const long row0 = loc.t0 + (long)loc.c * kC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the compute threads' gate loads go out before the setup below (their
    // latency is the first thing a chunk waits for)
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;              // TMEM lane of a compute thread
    const RowGates gates = warp > 0 ? load_gates(a, row0, lenc, h, r) : RowGates{0.f, 0.f, 1.f};

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + PS_BAR);
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(sm + PS_TMEMPTR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + PS_FLAGS);
    float *g_s = reinterpret_cast<float *>(sm + PS_G);
    const float *b_s = g_s + 64, *bg_s = g_s + 128, *eg_s = g_s + 256;

    const int r0 = (int)row0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kPrepBars; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
        // K and Q before the rest of the setup (their latency heads the chunk's
        // chain); V once the solve has freed A's region (the load overlaps the
        // T images, W and its extraction)
        mbar_arrive_expect_tx(&bars[PB_FULL], 32768);
        tma_load_3d(sm + PS_K, &maps.k, &bars[PB_FULL], 0, h, r0);
        tma_load_3d(sm + PS_K + 8192, &maps.k, &bars[PB_FULL], 64, h, r0);
        tma_load_3d(sm + PS_Q, &maps.q, &bars[PB_FULL], 0, h, r0);
        tma_load_3d(sm + PS_Q + 8192, &maps.q, &bars[PB_FULL], 64, h, r0);
    }
    if (warp == 0) {
        tmem_alloc(tmem_ptr, kPrepTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    uint8_t *img = a.workspace_chunks + ((size_t)gc * H + h) * a.chunk_bytes;

    // Warp 0 allocated TMEM and (thread 0) issued the tile loads; compute thread 0
    // issues the MMAs and the V load itself, where its warps' work makes them
    // ready (no hand-off through another warp), and drains them at the end.
    if (warp > 0) {
        const int cw = threadIdx.x - 32;
        // rows ta, ta + 8 and column pairs 8 kb + j2 of the M=64 accumulators (16x256b loads)
        const int ta = 16 * q4 + (lane >> 2), j2 = 2 * (lane & 3);
        const uint32_t tq = tmem + ((uint32_t)(32 * q4) << 16);
        float *Af = reinterpret_cast<float *>(sm + PS_AF);
        float *Tf = reinterpret_cast<float *>(sm + PS_TF);
        float *Xs = reinterpret_cast<float *>(sm + PS_XS);
        // MMA operands (shared-memory addresses) and instruction descriptors
        const uint32_t kk_ = smem_u32(sm + PS_K), qq = smem_u32(sm + PS_Q), vv = smem_u32(sm + PS_V);
        const uint32_t tbg = smem_u32(sm + PS_TBG), tb = smem_u32(sm + PS_TB);
        constexpr uint32_t ID_KK = idesc_bf16(64, 64, 0, 0);
        constexpr uint32_t ID_W = idesc_bf16(64, 128, 0, 1);
        const uint32_t ID_U = Dv == 128 ? idesc_bf16(64, 128, 0, 1) : idesc_bf16(64, 64, 0, 1);
        bool v_issued = false;           // compute thread 0's: copies and MMAs to drain

        if constexpr (CH) {
            prep_channel_front(a, sm, g_s, gates, cw, r, lenc, row0, h, img, bars, abort_flag);
        } else {
        chunk_gates(gates, r, lane, g_s);
        if (cw == 0 && wait_bar(&bars[PB_FULL], 0, abort_flag, a.err, a.wait_ns)) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {     // K K^T: A = B = the K tile (K-major)
                const uint32_t off = (kk >> 2) * 8192 + (kk & 3) * 32;
                mma_bf16(tmem + PT_KK, smem_desc(kk_ + off, 16, 1024, kSw128),
                         smem_desc(kk_ + off, 16, 1024, kSw128), ID_KK, kk > 0);
            }
            mma_commit(&bars[PB_KK]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {     // Q K^T: A = the Q tile, B = the K tile (K-major)
                const uint32_t off = (kk >> 2) * 8192 + (kk & 3) * 32;
                mma_bf16(tmem + PT_QK, smem_desc(qq + off, 16, 1024, kSw128),
                         smem_desc(kk_ + off, 16, 1024, kSw128), ID_KK, kk > 0);
            }
            mma_commit(&bars[PB_QK]);
            if (!wait_bar(&bars[PB_KK], 0, abort_flag, a.err, a.wait_ns)) *abort_flag = 1;
        }
        named_bar_sync(1, 128);
        if (!*abort_flag) {
            tc_fence_after();
            // A rows ta, ta + 8: beta_t (K K^T)[t][s] e^{g_t - g_s}, s < t
            float v[32];
            gram_rows<true>(tq + PT_KK, ta, lane, b_s, g_s, v);
#pragma unroll
            for (int kb = 0; kb < 8; ++kb) {
                const int s = 8 * kb + j2;
                *reinterpret_cast<float2 *>(Af + ta * kLd + s) = make_float2(v[4 * kb], v[4 * kb + 1]);
                *reinterpret_cast<float2 *>(Af + (ta + 8) * kLd + s) = make_float2(v[4 * kb + 2], v[4 * kb + 3]);
            }
            tc_fence_before();
        }
        if (cw == 0 && !*abort_flag && !wait_bar(&bars[PB_QK], 0, abort_flag, a.err, a.wait_ns)) *abort_flag = 1;
        named_bar_sync(1, 128);
        if (!*abort_flag) {
            // the Q tile landed before the Q K^T product was issued; this wait (complete
            // already) makes the copy visible to these threads
            wait_bar(&bars[PB_FULL], 0, abort_flag, a.err, a.wait_ns);
            tc_fence_after();
            // P rows ta, ta + 8: (Q K^T)[t][s] e^{g_t - g_s}, s <= t -> bf16 K-major
            // SW128 image, stored from registers
            float v[32];
            gram_rows<false>(tq + PT_QK, ta, lane, nullptr, g_s, v);
            uint8_t *pi = img + kImgP + 2 * j2;
#pragma unroll
            for (int kb = 0; kb < 8; ++kb) {
                *reinterpret_cast<uint32_t *>(pi + swz(ta, kb, 128)) = pack_bf16(v[4 * kb], v[4 * kb + 1]);
                *reinterpret_cast<uint32_t *>(pi + swz(ta + 8, kb, 128)) = pack_bf16(v[4 * kb + 2], v[4 * kb + 3]);
            }
            tc_fence_before();
        }
        }
        named_bar_sync(1, 128);      // Q is dead: T goes there
        if (!*abort_flag) {
            ut_solve(Af, Tf, Xs, cw);      // ends with a barrier: A is dead from here
            // T diag(beta e^g) and T diag(beta gamma) as bf16 K-major SW128 images,
            // over T: every thread reads its part of T before any image is written
            const int t = cw >> 1, half = cw & 1;
            uint4 y1[4], y2[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int s0 = 32 * half + 8 * cc;
                const float4 t0 = *reinterpret_cast<const float4 *>(Tf + t * kLd + s0);
                const float4 t1 = *reinterpret_cast<const float4 *>(Tf + t * kLd + s0 + 4);
                const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                float z1[8], z2[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    z1[e] = CH ? tv[e] * b_s[s0 + e] : tv[e] * b_s[s0 + e] * eg_s[s0 + e];
                    z2[e] = tv[e] * bg_s[s0 + e];
                }
                y1[cc] = pack8(z1);
                y2[cc] = pack8(z2);
            }
            named_bar_sync(1, 128);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                *reinterpret_cast<uint4 *>(sm + PS_TBG + swz(t, 4 * half + cc, 128)) = y1[cc];
                *reinterpret_cast<uint4 *>(sm + PS_TB + swz(t, 4 * half + cc, 128)) = y2[cc];
            }
        }
        // generic accesses to A's region (reused by the V load) and the T images
        // (read by the MMAs) before the async proxy touches them
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (cw == 0 && !*abort_flag) {
            // V into A's region (dead since the solve; the fence above ordered the
            // generic accesses to it), then W = T diag(beta e^g) K  (B = K, MN-major)
            mbar_arrive_expect_tx(&bars[PB_VFULL], 64 * Dv * 2);
            tma_load_3d(sm + PS_V, &maps.v, &bars[PB_VFULL], 0, h, r0);
            if (Dv == 128) tma_load_3d(sm + PS_V + 8192, &maps.v, &bars[PB_VFULL], 64, h, r0);
            v_issued = true;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + PT_W, smem_desc(tbg + kk * 32, 16, 1024, kSw128),
                         smem_desc(kk_ + kk * 2048, 8192, 1024, kSw128), ID_W, kk > 0);
            mma_commit(&bars[PB_W]);
            if (!wait_bar(&bars[PB_W], 0, abort_flag, a.err, a.wait_ns)) *abort_flag = 1;
        }
        named_bar_sync(1, 128);
        if (!*abort_flag) {
            tc_fence_after();
            // -W rows -> bf16 K-major SW128 image (2 halves of 64 columns), over K
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld_16x256b_x4(tq + PT_W + 64 * half, v);
                tmem_ld_16x256b_x4(tq + PT_W + 64 * half + 32, v + 16);
                tmem_wait_ld();
                uint8_t *wi = sm + PS_WIMG + half * 8192 + 2 * j2;
#pragma unroll
                for (int kb = 0; kb < 8; ++kb) {
                    *reinterpret_cast<uint32_t *>(wi + swz(ta, kb, 128)) = pack_bf16(-v[4 * kb], -v[4 * kb + 1]);
                    *reinterpret_cast<uint32_t *>(wi + swz(ta + 8, kb, 128)) =
                        pack_bf16(-v[4 * kb + 2], -v[4 * kb + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
        }
        named_bar_sync(1, 128);
        if (cw == 0 && !*abort_flag) {
            bulk_store(img + kImgW, sm + PS_WIMG, 16384);
            bulk_commit();
            // U' = T diag(beta gamma) V  (B = V, MN-major), into the columns W has left
            if (wait_bar(&bars[PB_VFULL], 0, abort_flag, a.err, a.wait_ns)) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + PT_U, smem_desc(tb + kk * 32, 16, 1024, kSw128),
                             smem_desc(vv + kk * 2048, 8192, 1024, kSw128), ID_U, kk > 0);
                mma_commit(&bars[PB_U]);
                if (!wait_bar(&bars[PB_U], 0, abort_flag, a.err, a.wait_ns)) *abort_flag = 1;
            }
        }
        named_bar_sync(1, 128);
        if (!*abort_flag) {
            tc_fence_after();
            // U' rows -> bf16, value slices of width NV: slice s at s*64*NV*2, row t at t*NV*2
            for (int half = 0; half < Dv / 64; ++half) {
                float v[32];
                tmem_ld_16x256b_x4(tq + PT_U + 64 * half, v);
                tmem_ld_16x256b_x4(tq + PT_U + 64 * half + 32, v + 16);
                tmem_wait_ld();
#pragma unroll
                for (int kb = 0; kb < 8; ++kb) {
                    const int col = 64 * half + 8 * kb + j2;
                    uint8_t *ui = sm + PS_UIMG + (col / NV) * (64 * NV * 2) + (col % NV) * 2;
                    *reinterpret_cast<uint32_t *>(ui + ta * (NV * 2)) = pack_bf16(v[4 * kb], v[4 * kb + 1]);
                    *reinterpret_cast<uint32_t *>(ui + (ta + 8) * (NV * 2)) = pack_bf16(v[4 * kb + 2], v[4 * kb + 3]);
                }
            }
            fence_proxy_async_smem();
        }
        named_bar_sync(1, 128);
        if (cw == 0) {
            if (!*abort_flag) {
                bulk_store(img + kImgU, sm + PS_UIMG, 64 * Dv * 2);
                bulk_store(img + img_decay(Dv), eg_s, CH ? 1024 : 512);     // e^g, e^{g_C - g} (, e^{G_C})
                bulk_commit();
            }
            bulk_wait_reads();
            // the CTA may not exit (nor free TMEM) with copies or MMAs in flight
            mma_commit(&bars[PB_DRAIN]);
            drain_bar(&bars[PB_DRAIN], 0, a.wait_ns);
            drain_bar(&bars[PB_FULL], 0, a.wait_ns);
            if (v_issued) drain_bar(&bars[PB_VFULL], 0, a.wait_ns);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kPrepTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Kernel 2: scan.  One CTA per (sequence, head, value slice of width NV).
//
// The chunk-to-chunk dependency is S -> U = U' - W S -> S' = e^{g_C} S + K^T U~,
// two small dependent products per chunk (64x128 by 128xNV, then 128x64 by
// 64xNV).  On tcgen05 each such instruction costs about 90 cycles of pipe
// time whatever its size, plus a commit round trip, so this latency-bound
// chain runs on register-fragment tensor-core MMAs (mma.sync m16n8k16, bf16
// in, fp32 accumulate) with ldmatrix operands.  The outputs of the chunk's
// rows come out of the same pass: Q S with the operand fragments of S that U
// uses (rows then scaled by e^{g_t}), and P U once U is in shared memory.
//   warps 0..3  warp w owns key rows 32w..32w+31 of the fp32 state (as
//               accumulator fragments) and token rows 16w..16w+15 of U and O,
//               across the slice's NV value columns (splitting the columns
//               over twice the warps doubles the operand traffic through
//               shared memory and measured slower)
//   warp 4      producer: the K and Q tiles by TMA, -W, P, U' and the decay
//               factors by bulk copies, into a 3-stage ring.
// ---------------------------------------------------------------------------
constexpr int kScanWarps = 4;
constexpr int kScanThreads = (kScanWarps + 1) * 32;
constexpr int kScanStages = 3;
// per-stage shared memory (bytes): -W 16K | K 16K | Q 16K | P 8K | U' <= 4K | decay 512
constexpr uint32_t SS_W = 0, SS_K = 16384, SS_Q = 32768, SS_P = 49152, SS_U = 57344, SS_G = 61440;
constexpr uint32_t SS_STAGE = 62464;                          // multiple of 1024
enum ScanBar { SB_FULL = 0, SB_EMPTY = kScanStages, kScanBars = 2 * kScanStages };
// then: state [128][RS] bf16, U~ [64][RS], U [64][RS], barriers, flags (RS = 2 NV + 16)
template <int NV> struct ScanSmem {
    static constexpr uint32_t RS = NV * 2 + 16;
    static constexpr uint32_t SS = kScanStages * SS_STAGE;
    static constexpr uint32_t UT = SS + 128 * RS;
    static constexpr uint32_t UU = UT + 64 * RS;       // U (unscaled), the B operand of P U
    static constexpr uint32_t BAR = UU + 64 * RS;
    static constexpr uint32_t FLAGS = BAR + kScanBars * 8;
    static constexpr uint32_t BYTES = FLAGS + 16 + 1024;
};

struct ScanMaps {
    CUtensorMap k, q;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t *r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t *r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t *r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(addr));
}
// D += A(16x16, row) * B(16x8, col): bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma16816(float *d, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// ldmatrix row address for the 16x16 tile at (row0, col0) of a bf16 K-major
// SW128 image (64-column halves of `halfbytes`, 128-byte rows).  Lane i
// addresses row (i&7) + 8((i>>3)&1), column block (i>>4).
__device__ __forceinline__ uint32_t a_addr_sw128(uint32_t base, int row0, int col0, int lane, uint32_t halfbytes) {
    const int row = row0 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const int col = col0 + 8 * (lane >> 4);
    return base + (col >> 6) * halfbytes + swz(row, (col & 63) >> 3, 128);
}
// ldmatrix.trans address giving the A fragment of the transpose of a
// K-major SW128 image: element (m, k) of the fragment is image[k][m].
__device__ __forceinline__ uint32_t at_addr_sw128(uint32_t base, int m0, int k0, int lane, uint32_t halfbytes) {
    const int mi = lane >> 3;
    const int row = k0 + (lane & 7) + 8 * (mi >> 1);     // image row = k
    const int col = m0 + 8 * (mi & 1);                   // image column = m
    return base + (col >> 6) * halfbytes + swz(row, (col & 63) >> 3, 128);
}
// ldmatrix.trans address for B fragments of a row-major [k][n] bf16 buffer
// (row stride rs bytes): x4 gives n0..n0+7 and n0+8..n0+15, x2 gives n0..n0+7.
__device__ __forceinline__ uint32_t b_addr_rm(uint32_t base, int k0, int n0, int lane, uint32_t rs) {
    const int row = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const int col = n0 + 8 * (lane >> 4);
    return base + row * rs + col * 2;
}
// B fragments for one warp's NW value columns (8, 16 or 32) at k-tile k0:
// bf[2nt], bf[2nt+1] feed n-tile nt.
template <int NW>
__device__ __forceinline__ void ld_b(uint32_t base, int k0, int n0, int lane, uint32_t rs, uint32_t *bf) {
    if constexpr (NW == 8) {
        ldsm_x2_t(b_addr_rm(base, k0, n0, lane & 15, rs), bf);
    } else {
#pragma unroll
        for (int i = 0; i < NW / 16; ++i) ldsm_x4_t(b_addr_rm(base, k0, n0 + 16 * i, lane, rs), bf + 4 * i);
    }
}

template <int NV, bool CH>
__global__ void __launch_bounds__(kScanThreads, 1)
scan_kernel(const __grid_constant__ ScanMaps maps, const PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_align_1024(smem_raw);
    using L = ScanSmem<NV>;
    constexpr uint32_t SC_SS = L::SS, SC_UT = L::UT;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::FLAGS);
    volatile int *agent_flag = abort_flag + 1;     // the producer's
    constexpr int NW = NV * 4 / kScanWarps;     // value columns per warp
    constexpr int NT = NW / 8;                  // n-tiles of 8 columns per warp
    constexpr uint32_t RS = NV * 2 + 16;        // padded row stride of the S / U~ buffers
    constexpr uint32_t UBYTES = 64 * NV * 2;    // U' slice bytes
    constexpr uint32_t NCW = kScanWarps * 32;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tg = lane & 3;
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
    const float *s_in = a.s0;
    float *s_out = a.sf;
    const int j0 = slice * NV;
    const int H = a.H, Dv = a.Dv;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kScanStages; ++i) {
            mbar_init(&bars[SB_FULL + i], 1);
            mbar_init(&bars[SB_EMPTY + i], NCW);
        }
        *abort_flag = 0;
        *agent_flag = 0;
        fence_mbar_init();
        if (nchunks > 0) prefetch_tensormap(&maps.k);
    }
    __syncthreads();
    const uint32_t smb = smem_u32(sm);

    if (warp == kScanWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            pdl_wait_primary();      // the prep's images are complete and visible
            int last[kScanStages];   // last chunk whose loads went out on each stage
            for (int i = 0; i < kScanStages; ++i) last[i] = -1;
            for (int c = 0; c < nchunks; ++c) {
                const int st = c % kScanStages;
                if (c >= kScanStages &&
                    !wait_bar2(&bars[SB_EMPTY + st], (c / kScanStages - 1) & 1, abort_flag, agent_flag, a.err, a.wait_ns))
                    break;
                if (c == a.debug_drop_chunk) continue;   // fault injection (tests only): never filled
                last[st] = c;
                uint64_t *full = &bars[SB_FULL + st];
                uint8_t *stg = sm + st * SS_STAGE;
                const uint8_t *img = a.workspace_chunks + ((size_t)(gc0 + c) * H + h) * a.chunk_bytes;
                constexpr uint32_t GBYTES = CH ? 1024 : 512;
                mbar_arrive_expect_tx(full, 16384 * 3 + 8192 + UBYTES + GBYTES);
                if constexpr (CH) {
                    // per-channel decay: the prep's K o e^{G_C - G} and Q o e^{G} images
                    bulk_load(stg + SS_K, img + img_kt(Dv), 16384, full);
                    bulk_load(stg + SS_Q, img + img_qt(Dv), 16384, full);
                } else {
                    const int r0 = (int)(t0 + (long)c * kC);
                    tma_load_3d(stg + SS_K, &maps.k, full, 0, h, r0);
                    tma_load_3d(stg + SS_K + 8192, &maps.k, full, 64, h, r0);
                    tma_load_3d(stg + SS_Q, &maps.q, full, 0, h, r0);
                    tma_load_3d(stg + SS_Q + 8192, &maps.q, full, 64, h, r0);
                }
                bulk_load(stg + SS_W, img + kImgW, 16384, full);
                bulk_load(stg + SS_P, img + kImgP, 8192, full);
                bulk_load(stg + SS_U, img + kImgU + (size_t)slice * UBYTES, UBYTES, full);
                bulk_load(stg + SS_G, img + img_decay(Dv), GBYTES, full);
            }
            // the CTA may not exit with copies in flight: after an abort the scan
            // warps stop consuming, so wait (bounded) for every stage's last fill
            for (int i = 0; i < kScanStages; ++i)
                if (last[i] >= 0) drain_bar(&bars[SB_FULL + i], (last[i] / kScanStages) & 1, a.wait_ns);
        }
        return;
    }

    // ---------------------------------------------------------------- scan warps
    const int rg = warp & 3;                    // row group
    const int c0 = (warp >> 2) * NW;            // first value column (within the slice)
    static_assert(kScanWarps == 4 || kScanWarps == 8, "warps cover 4 row groups");
    const int tid = threadIdx.x;
    // S fragments: rows d = 32rg + 16mt + g (+8), columns c0 + 8nt + 2tg (+1)
    float S[2][NT][4];
    const size_t sb = ((size_t)n * H + h) * kDK * Dv + j0;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int d = 32 * rg + 16 * mt + g + 8 * hh, j = c0 + 8 * nt + 2 * tg;
                float2 x = make_float2(0.f, 0.f);
                if (s_in) x = *reinterpret_cast<const float2 *>(s_in + sb + (size_t)d * Dv + j);
                S[mt][nt][2 * hh] = x.x;
                S[mt][nt][2 * hh + 1] = x.y;
            }
    const uint32_t ssb = smb + SC_SS, utb = smb + SC_UT;
    for (int c = 0; c < nchunks; ++c) {
        const int st = c % kScanStages;
        const uint32_t stg = smb + st * SS_STAGE;
        const float *eg_s = reinterpret_cast<const float *>(sm + st * SS_STAGE + SS_G);
        const float *ed_s = eg_s + 64;
        // ---- S -> bf16: row-major [d][j] in shared memory (the B operand below)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int d = 32 * rg + 16 * mt + g + 8 * hh, j = c0 + 8 * nt + 2 * tg;
                    const uint32_t v = pack_bf16(S[mt][nt][2 * hh], S[mt][nt][2 * hh + 1]);
                    *reinterpret_cast<uint32_t *>(sm + SC_SS + d * RS + j * 2) = v;
                }
        if (tid == 0 && !wait_bar(&bars[SB_FULL + st], (c / kScanStages) & 1, abort_flag, a.err, a.wait_ns)) *abort_flag = 1;
        named_bar_sync(1, NCW);
        if (*abort_flag) break;
        // ---- U = U' + (-W) S for rows t = 16rg .. 16rg+15 (accumulators start at U')
        const int ta = 16 * rg + g, tb = ta + 8;
        const uint8_t *up = sm + st * SS_STAGE + SS_U;
        float acc[2][NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int j = c0 + 8 * nt + 2 * tg;
            const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(up + (ta * NV + j) * 2));
            const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(up + (tb * NV + j) * 2));
            acc[0][nt][0] = fa.x; acc[0][nt][1] = fa.y; acc[0][nt][2] = fb.x; acc[0][nt][3] = fb.y;
            acc[1][nt][0] = acc[1][nt][1] = acc[1][nt][2] = acc[1][nt][3] = 0.f;
        }
        // O = diag(e^g) (Q S_c) (+ P U below) for the same rows: Q S_c shares the
        // state operand fragments with U
        float ao[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) ao[nt][0] = ao[nt][1] = ao[nt][2] = ao[nt][3] = 0.f;
        // operands of a group of k-steps are loaded before its MMAs are issued, so
        // the shared-memory latency is paid once per group
        constexpr int KGU = NW >= 32 ? 2 : 4;
#pragma unroll
        for (int k0 = 0; k0 < 8; k0 += KGU) {
            uint32_t af[KGU][4], aq[KGU][4], bf[KGU][NW / 4 > 4 ? NW / 4 : 4];
#pragma unroll
            for (int kk = 0; kk < KGU; ++kk) {
                ldsm_x4(a_addr_sw128(stg + SS_W, 16 * rg, 16 * (k0 + kk), lane, 8192), af[kk]);
                ld_b<NW>(ssb, 16 * (k0 + kk), c0, lane, RS, bf[kk]);
                ldsm_x4(a_addr_sw128(stg + SS_Q, 16 * rg, 16 * (k0 + kk), lane, 8192), aq[kk]);
            }
#pragma unroll
            for (int kk = 0; kk < KGU; ++kk)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma16816(acc[kk & 1][nt], af[kk], bf[kk][2 * nt], bf[kk][2 * nt + 1]);
                    mma16816(ao[nt], aq[kk], bf[kk][2 * nt], bf[kk][2 * nt + 1]);
                }
        }
        if constexpr (!CH) {
            const float ea = eg_s[ta], eb = eg_s[tb];     // e^{g_t} (per-channel: inside Q's image)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                ao[nt][0] *= ea;
                ao[nt][1] *= ea;
                ao[nt][2] *= eb;
                ao[nt][3] *= eb;
            }
        }
        // ---- U and U~ = e^{g_C - g_t} U -> shared memory (B operands of P U and K^T U~;
        // per-channel: the factor is inside K's image and U~ = U)
        const float da = CH ? 1.f : ed_s[ta], db = CH ? 1.f : ed_s[tb];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int j = c0 + 8 * nt + 2 * tg;
            const float u0 = acc[0][nt][0] + acc[1][nt][0], u1 = acc[0][nt][1] + acc[1][nt][1];
            const float u2 = acc[0][nt][2] + acc[1][nt][2], u3 = acc[0][nt][3] + acc[1][nt][3];
            *reinterpret_cast<uint32_t *>(sm + L::UU + ta * RS + j * 2) = pack_bf16(u0, u1);
            *reinterpret_cast<uint32_t *>(sm + L::UU + tb * RS + j * 2) = pack_bf16(u2, u3);
            *reinterpret_cast<uint32_t *>(sm + SC_UT + ta * RS + j * 2) = pack_bf16(u0 * da, u1 * da);
            *reinterpret_cast<uint32_t *>(sm + SC_UT + tb * RS + j * 2) = pack_bf16(u2 * db, u3 * db);
        }
        named_bar_sync(1, NCW);
        // ---- S <- e^{g_C} S + K^T U~ for rows d = 32rg .. 32rg+31
        float ds[2][2][NT][4];
#pragma unroll
        for (int p2 = 0; p2 < 2; ++p2)
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    ds[p2][mt][nt][0] = ds[p2][mt][nt][1] = ds[p2][mt][nt][2] = ds[p2][mt][nt][3] = 0.f;
        constexpr int KGD = NW >= 32 ? 2 : 4;
#pragma unroll
        for (int k0 = 0; k0 < 4; k0 += KGD) {
            uint32_t af[KGD][2][4], bf[KGD][NW / 4 > 4 ? NW / 4 : 4];
#pragma unroll
            for (int kk = 0; kk < KGD; ++kk) {
                ld_b<NW>(utb, 16 * (k0 + kk), c0, lane, RS, bf[kk]);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
                    ldsm_x4_t(at_addr_sw128(stg + SS_K, 32 * rg + 16 * mt, 16 * (k0 + kk), lane, 8192), af[kk][mt]);
            }
#pragma unroll
            for (int kk = 0; kk < KGD; ++kk)
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma16816(ds[kk & 1][mt][nt], af[kk][mt], bf[kk][2 * nt], bf[kk][2 * nt + 1]);
        }
        const float *dC = eg_s + 128;                 // per-channel: e^{G_C} of each key dim
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float eC = CH ? dC[32 * rg + 16 * mt + g + 8 * (i >> 1)] : eg_s[63];     // e^{g_C}
                    S[mt][nt][i] = fmaf(eC, S[mt][nt][i], ds[0][mt][nt][i] + ds[1][mt][nt][i]);
                }
        // ---- O += P U for rows t = 16rg .. 16rg+15, then the store (masked tail)
        {
            const uint32_t uub = smb + L::UU;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t ap[4], bu[NW / 4 > 4 ? NW / 4 : 4];
                ldsm_x4(a_addr_sw128(stg + SS_P, 16 * rg, 16 * kk, lane, 8192), ap);
                ld_b<NW>(uub, 16 * kk, c0, lane, RS, bu);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma16816(ao[nt], ap, bu[2 * nt], bu[2 * nt + 1]);
            }
        }
        mbar_arrive(&bars[SB_EMPTY + st]);
        {
            const int lenc = (int)min((long)kC, len - (long)c * kC);
            __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(a.out) + ((size_t)(t0 + (long)c * kC) * H + h) * Dv + j0;
            const float sc = a.scale;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int j = c0 + 8 * nt + 2 * tg;
                if (ta < lenc)
                    *reinterpret_cast<uint32_t *>(ob + (size_t)ta * H * Dv + j) = pack_bf16(sc * ao[nt][0], sc * ao[nt][1]);
                if (tb < lenc)
                    *reinterpret_cast<uint32_t *>(ob + (size_t)tb * H * Dv + j) = pack_bf16(sc * ao[nt][2], sc * ao[nt][3]);
            }
        }
        // No barrier here: the next chunk writes the state buffer after every
        // warp passed this chunk's second barrier (its reads of the state are
        // done), and U~ after the next first barrier (every warp is past this
        // chunk's update).
    }
    if (s_out && !*abort_flag) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int d = 32 * rg + 16 * mt + g + 8 * hh, j = c0 + 8 * nt + 2 * tg;
                    *reinterpret_cast<float2 *>(s_out + sb + (size_t)d * Dv + j) =
                        make_float2(S[mt][nt][2 * hh], S[mt][nt][2 * hh + 1]);
                }
    }
}

// ---------------------------------------------------------------------------
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
    // The scan is bound by MMA throughput per SM: narrow slices spread a head
    // over more SMs; widen them once the SMs are covered.
    return units * (Dv / 32) >= 148 ? 32 : 16;
}

template <int NV, bool CH>
cudaError_t init_attrs() {
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [] {
        attr = set_smem(prep_kernel<NV, CH>, CH ? kPrepSmemCh : kPrepSmem);
        if (attr == cudaSuccess) attr = set_smem(scan_kernel<NV, CH>, ScanSmem<NV>::BYTES);
    });
    return attr;
}

template <int NV, bool CH>
cudaError_t launch_nv(const PrefillArgs &a, long chunks_grid, cudaStream_t s) {
    cudaError_t e = init_attrs<NV, CH>();
    if (e != cudaSuccess) return e;
    PrepMaps pm;
    ScanMaps sm;
    std::memset(&pm, 0, sizeof(pm));
    std::memset(&sm, 0, sizeof(sm));
    if (a.total_T > 0) {
        if (!make_map(&pm.q, a.q, kDK, a.H, a.total_T, 64) || !make_map(&pm.k, a.k, kDK, a.H, a.total_T, 64) ||
            !make_map(&pm.v, a.v, a.Dv, a.H, a.total_T, 64))
            return cudaErrorInvalidValue;
        sm.k = pm.k;
        sm.q = pm.q;
    }
    const dim3 scan_grid(a.Dv / NV, a.H, a.num_seqs);
    const uint32_t scan_smem = ScanSmem<NV>::BYTES;
    const dim3 chunk_grid((unsigned)chunks_grid, a.H, 1);

    if (chunks_grid > 0) {
        prep_kernel<NV, CH><<<chunk_grid, kPrepThreads, CH ? kPrepSmemCh : kPrepSmem, s>>>(pm, a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // programmatic stream serialization: the scan's launch and prologue overlap
    // the prep's last CTAs; only its producer waits for the prep to complete
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = scan_grid;
    cfg.blockDim = dim3(kScanThreads, 1, 1);
    cfg.dynamicSmemBytes = scan_smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = chunks_grid > 0 ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, scan_kernel<NV, CH>, sm, a);
}

// Bytes of one (chunk, head) image: -W, P, U', the decay factors; with a decay
// per key dim, e^{G_C} and the K and Q images too.
size_t image_bytes(int Dv, bool channel) {
    return channel ? (size_t)img_qt(Dv) + 16384 : (size_t)kImgU + 64 * (size_t)Dv * 2 + 512;
}

size_t header_bytes(int num_seqs) {
    size_t b = 4 * (size_t)(num_seqs + 1);
    return (b + 1023) / 1024 * 1024;
}

}  // namespace

bool chunked_supported(rda_dtype_t dtype, int Dk, int Dv) {
    return dtype == RDA_BF16 && Dk == kDK && (Dv == 64 || Dv == 128);
}

size_t chunked_workspace_bytes(long total_T, int T, int B, int H, int Dv, int num_seqs, bool channel) {
    long chunks;
    if (num_seqs > 0) chunks = (total_T + kC - 1) / kC + num_seqs;     // packed: upper bound
    else chunks = (long)B * ((T + kC - 1) / kC);
    return header_bytes(num_seqs) + (size_t)chunks * H * image_bytes(Dv, channel);
}

cudaError_t launch_chunked(const PrefillArgs &a0, void *scratch, cudaStream_t s) {
    PrefillArgs a = a0;
    uint8_t *ws = static_cast<uint8_t *>(scratch);
    const int nseq_hdr = a.cu_seqlens ? a.num_seqs : 0;
    a.workspace_chunks = ws + header_bytes(nseq_hdr);
    a.chunk_bytes = image_bytes(a.Dv, a.channel_decay);
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
    const bool wide = choose_nv(units, a.Dv) == 32;
    if (a.channel_decay)
        return wide ? launch_nv<32, true>(a, chunks_grid, s) : launch_nv<16, true>(a, chunks_grid, s);
    return wide ? launch_nv<32, false>(a, chunks_grid, s) : launch_nv<16, false>(a, chunks_grid, s);
}

}  // namespace rda
