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
// the HBM time of one decode step.  From three tokens (at Dk = Dv = 128) the
// products with the state and its update run on tf32 tensor-core MMAs with
// split operands (fp32 accuracy); below that, on paired fp32 FMAs.
#include <type_traits>

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

// ---------------------------------------------------------------------------
// Dk = Dv = 128 on the tensor cores.  Warp w holds value columns
// j0 = 16w .. 16w+15 of the state for every key dim, in the accumulator layout
// of an m16n8k8 tf32 MMA whose rows are value columns (row m <-> column
// j0 + 2(m%8) + m/8) and whose columns are key dims: for key block nb
// (dims 8nb .. 8nb+7), with d = 8nb + 2tg and j = j0 + 2g (g = lane/4, tg = lane%4),
//     s[nb] = { S[d][j], S[d+1][j], S[d][j+1], S[d+1][j+1] }
// so that each thread moves the state in pairs of adjacent columns.  The same
// registers, in the order {0, 2, 1, 3}, are the A operand of the products with
// the new keys and queries when the reduction index of block nb is read in the
// order 0,2,4,6,1,3,5,7 (A column tg is key dim d, column tg+4 is d+1; the B rows
// follow the same order), and the accumulator of the update
// S_new^T = c S^T + W K (M = value columns, K = tokens, N = key dims).  fp32
// accuracy from tf32 MMAs: every fp32 operand is split into a tf32 head and a
// tf32 tail (x = hi + lo + O(2^-22 |x|)) and hi*hi + lo*hi + hi*lo are
// accumulated in fp32; bf16 keys and queries are exact in tf32 (no tail).
// ---------------------------------------------------------------------------
constexpr int kTcD = 128;
constexpr int kTcKP = kTcD + 8;     // row stride of the key / query rows (conflict-free float2 B loads)
constexpr int kTcWP = kTcD + 4;     // row stride of the coefficient rows

__device__ __forceinline__ uint32_t tf32_of(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
    hi = tf32_of(x);
    lo = tf32_of(x - __uint_as_float(hi));
}
// D += A(16x8, row) * B(8x8, col), tf32 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_tf32_m16n8k8(float *d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                 uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// acc += a * b for an fp32 A fragment and a B fragment given as tf32 head / tail
// (no tail when EXACT_B).
template <bool EXACT_B>
__device__ __forceinline__ void mma_f32_split(float *acc, const float *a, uint32_t bh0, uint32_t bh1, uint32_t bl0,
                                              uint32_t bl1) {
    uint32_t ah[4], al[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) split_tf32(a[i], ah[i], al[i]);
    mma_tf32_m16n8k8(acc, ah[0], ah[1], ah[2], ah[3], bh0, bh1);
    mma_tf32_m16n8k8(acc, al[0], al[1], al[2], al[3], bh0, bh1);
    if (!EXACT_B) mma_tf32_m16n8k8(acc, ah[0], ah[1], ah[2], ah[3], bl0, bl1);
}

// Persistent form: each CTA loops over (sequence, head) units.  A unit's state
// (64 KiB) is copied into shared memory with 16-byte asynchronous copies
// (cp.async, completed by a hardware wait, no spin) and from there into the
// registers; the copy of the CTA's next unit is issued while the current one
// computes, so every SM always has state bytes in flight.  The next unit's rows
// and gates go out as soon as their buffer is free; its state by the 128
// threads that the token recurrence leaves idle (4,096 copies issued at once
// back up the load queue: ~3,200 cycles of a ~16,400-cycle unit when every
// thread issued them in the chain).
constexpr int kTcRow = kTcD + 4;    // padded smem row (528 B): conflict-free 8-byte fragment reads
constexpr uint32_t kTcStateBytes = kTcD * kTcRow * 4;
constexpr uint32_t kTcRawBytes = 3 * kMaxT * kTcD * 4;                    // k, q, v rows (fp32 at most)
constexpr uint32_t kTcSmem = kTcStateBytes + kTcRawBytes + 3 * kMaxT * 4; // + the gates

// Unit bh's state into shared memory: 4,096 16-byte pieces into the padded
// buffer, by `nthr` threads (thread index `tid` among them).
__device__ __forceinline__ void issue_unit_state(const DecodeArgs &a, int bh, uint32_t smem, int tid, int nthr) {
    const float *st = a.state + (size_t)bh * kTcD * kTcD;
    for (int id = tid; id < kTcD * kTcD / 4; id += nthr) {
        const int row = id >> 5, c16 = id & 31;
        cp_async16(smem + (row * kTcRow + c16 * 4) * 4, st + row * kTcD + c16 * 4);
    }
    cp_async_commit();
}
// The raw rows of unit bh's T keys, queries and values, and its gates (log
// alpha, beta, gamma), into shared memory.
template <typename Tio>
__device__ __forceinline__ void issue_unit_rows(const DecodeArgs &a, int bh, uint32_t smem) {
    const int T = a.T, H = a.H, b = bh / H, h = bh % H;
    constexpr int PR = kTcD * (int)sizeof(Tio) / 16;      // 16-byte pieces per row
    const uint32_t raw = smem + kTcStateBytes;
    for (int id = threadIdx.x; id < 3 * T * PR; id += kThreads) {
        const int which = id / (T * PR), t = (id / PR) % T, c = id % PR;
        const Tio *src = static_cast<const Tio *>(which == 0 ? a.k : (which == 1 ? a.q : a.v)) +
                         (((size_t)b * T + t) * H + h) * kTcD;
        cp_async16(raw + ((which * kMaxT + t) * kTcD) * (uint32_t)sizeof(Tio) + c * 16, reinterpret_cast<const char *>(src) + c * 16);
    }
    if (threadIdx.x < 3 * T) {
        const int which = threadIdx.x / T, t = threadIdx.x % T;
        const float *src = which == 0 ? a.log_alpha : (which == 1 ? a.beta : a.gamma);
        if (src) cp_async4(raw + kTcRawBytes + (which * kMaxT + t) * 4, src + ((size_t)b * T + t) * H + h);
    }
    cp_async_commit();
}

template <typename Tio>
__global__ void __launch_bounds__(kThreads, 2)
decode_tokens_tc_kernel(DecodeArgs a) {
    constexpr int D = kTcD;
    constexpr bool kExact = !std::is_same<Tio, float>::value;    // bf16 keys / queries are tf32-exact
    __shared__ __align__(16) float k_s[kMaxT][kTcKP];      // k_t[d], rows past T zero
    __shared__ __align__(16) float q_s[kMaxT][kTcKP];
    __shared__ float v_s[kMaxT][D];                        // v_t (times gamma_t below)
    __shared__ __align__(16) float ab_s[2][kMaxT][D];      // a_t = s_0 . k_t, b_t = s_0 . q_t per column
    __shared__ float w_s[kMaxT][kTcWP];                    // final coefficients w_t per column, rows past T zero
    __shared__ float gp_s[kThreads / 32][2][kMaxT][kMaxT]; // Gram partials per warp (16 key dims each)
    __shared__ float kk_s[kMaxT][kMaxT];                   // [i][t] = k_i . k_t
    __shared__ float kq_s[kMaxT][kMaxT];                   // [i][t] = k_i . q_t
    __shared__ float g_s[3][kMaxT];                        // alpha, beta, gamma
    __shared__ float c_s;

    extern __shared__ __align__(16) float sbuf[];         // [kTcD][kTcRow] state of the current unit

    const int T = a.T, H = a.H;
    const int units = a.B * H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tg = lane & 3;
    const int jc = 16 * warp + 2 * g;                      // this thread's column pair
    const uint32_t buf = static_cast<uint32_t>(__cvta_generic_to_shared(sbuf));
    const Tio *raw_s = reinterpret_cast<const Tio *>(reinterpret_cast<const char *>(sbuf) + kTcStateBytes);
    const float *graw_s = reinterpret_cast<const float *>(reinterpret_cast<const char *>(sbuf) + kTcStateBytes +
                                                          kTcRawBytes);
    if ((int)blockIdx.x < units) {
        issue_unit_rows<Tio>(a, blockIdx.x, buf);
        issue_unit_state(a, blockIdx.x, buf, threadIdx.x, kThreads);
    }
    for (int bh = blockIdx.x; bh < units; bh += gridDim.x) {
        const int b = bh / H, h = bh % H;
        float *st = a.state + (size_t)bh * D * D;
        auto tok = [&](int t) { return ((size_t)b * T + t) * H + h; };
        // this unit's copies have landed: state -> registers, rows and gates ->
        // the fp32 work arrays; then the next unit's copy
        cp_async_wait_all();
        __syncthreads();
        float s[16][4];
#pragma unroll
        for (int nb = 0; nb < 16; ++nb) {
            const float *p = sbuf + (8 * nb + 2 * tg) * kTcRow + jc;
            const float2 r0 = *reinterpret_cast<const float2 *>(p);
            const float2 r1 = *reinterpret_cast<const float2 *>(p + kTcRow);
            s[nb][0] = r0.x;
            s[nb][2] = r0.y;
            s[nb][1] = r1.x;
            s[nb][3] = r1.y;
        }
        if (threadIdx.x < kMaxT) {
            const int t = threadIdx.x;
            const bool live = t < T;
            g_s[0][t] = live ? expf(graw_s[t]) : 1.f;
            g_s[1][t] = live ? graw_s[kMaxT + t] : 0.f;
            g_s[2][t] = live && a.gamma ? graw_s[2 * kMaxT + t] : 1.f;
        }
        for (int i = threadIdx.x; i < kMaxT * D; i += kThreads) {
            const int t = i / D, d = i % D;
            const bool live = t < T;
            k_s[t][d] = live ? Io<Tio>::ld(raw_s + (0 * kMaxT + t) * D + d) : 0.f;
            q_s[t][d] = live ? Io<Tio>::ld(raw_s + (1 * kMaxT + t) * D + d) : 0.f;
            if (live) v_s[t][d] = Io<Tio>::ld(raw_s + (2 * kMaxT + t) * D + d);
        }
        __syncthreads();
        const bool has_next = bh + (int)gridDim.x < units;
        if (has_next) issue_unit_rows<Tio>(a, bh + gridDim.x, buf);
        __syncthreads();

        {
            // a_t and b_t for this warp's 16 columns: S^T [k q] over the 128 key dims
            // (B column n = token g; rows of block nb in the order of the A columns)
            float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int nb = 0; nb < 16; ++nb) {
                const float af[4] = {s[nb][0], s[nb][2], s[nb][1], s[nb][3]};
                const float2 kb = *reinterpret_cast<const float2 *>(&k_s[g][8 * nb + 2 * tg]);
                const float2 qb = *reinterpret_cast<const float2 *>(&q_s[g][8 * nb + 2 * tg]);
                uint32_t kh0, kl0, kh1, kl1, qh0, ql0, qh1, ql1;
                split_tf32(kb.x, kh0, kl0);
                split_tf32(kb.y, kh1, kl1);
                split_tf32(qb.x, qh0, ql0);
                split_tf32(qb.y, qh1, ql1);
                mma_f32_split<kExact>(pk, af, kh0, kh1, kl0, kl1);
                mma_f32_split<kExact>(pq, af, qh0, qh1, ql0, ql1);
            }
            // accumulator: column jc (+1), token 2tg (+1)
            if (2 * tg < T) {
                ab_s[0][2 * tg][jc] = pk[0];
                ab_s[0][2 * tg][jc + 1] = pk[2];
                ab_s[1][2 * tg][jc] = pq[0];
                ab_s[1][2 * tg][jc + 1] = pq[2];
            }
            if (2 * tg + 1 < T) {
                ab_s[0][2 * tg + 1][jc] = pk[1];
                ab_s[0][2 * tg + 1][jc + 1] = pk[3];
                ab_s[1][2 * tg + 1][jc] = pq[1];
                ab_s[1][2 * tg + 1][jc + 1] = pq[3];
            }
            // token Gram values over this warp's 16 key dims: K [K Q]^T (A rows = tokens
            // g; rows g + 8 zero)
            float gk[4] = {0.f, 0.f, 0.f, 0.f}, gq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 2 * warp; ks < 2 * warp + 2; ++ks) {
                const float af[4] = {k_s[g][8 * ks + tg], 0.f, k_s[g][8 * ks + tg + 4], 0.f};
                uint32_t kh0, kl0, kh1, kl1, qh0, ql0, qh1, ql1;
                split_tf32(k_s[g][8 * ks + tg], kh0, kl0);
                split_tf32(k_s[g][8 * ks + tg + 4], kh1, kl1);
                split_tf32(q_s[g][8 * ks + tg], qh0, ql0);
                split_tf32(q_s[g][8 * ks + tg + 4], qh1, ql1);
                mma_f32_split<kExact>(gk, af, kh0, kh1, kl0, kl1);
                mma_f32_split<kExact>(gq, af, qh0, qh1, ql0, ql1);
            }
            gp_s[warp][0][g][2 * tg] = gk[0];
            gp_s[warp][0][g][2 * tg + 1] = gk[1];
            gp_s[warp][1][g][2 * tg] = gq[0];
            gp_s[warp][1][g][2 * tg + 1] = gq[1];
        }
        __syncthreads();
        if (threadIdx.x < 2 * kMaxT * kMaxT) {
            const int which = threadIdx.x >> 6, i = (threadIdx.x >> 3) & 7, t = threadIdx.x & 7;
            float x = 0.f;
#pragma unroll
            for (int w = 0; w < kThreads / 32; ++w) x += gp_s[w][which][i][t];
            (which ? kq_s : kk_s)[i][t] = x;
        }
        __syncthreads();

        // the token recurrence, one value column per thread
        if (threadIdx.x < D) {
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
                w[t] = g_s[1][t] * (g_s[2][t] * v_s[t][j] - al * p);
                c *= al;
                float o = c * ab_s[1][t][j];
#pragma unroll
                for (int i = 0; i <= t; ++i) o = fmaf(w[i], kq_s[i][t], o);
                Io<Tio>::st(static_cast<Tio *>(a.out) + tok(t) * D + j, a.scale * o);
            }
#pragma unroll
            for (int t = 0; t < kMaxT; ++t) w_s[t][j] = t < T ? w[t] : 0.f;
            if (j == 0) c_s = c;
        } else if (has_next) {
            // the next unit's state, by the threads the recurrence leaves idle (its
            // buffer has been free since this unit's state moved into registers)
            issue_unit_state(a, bh + gridDim.x, buf, threadIdx.x - D, kThreads - D);
        }
        __syncthreads();

        // S_new^T = c S^T + W K: A = W (value columns x tokens), B = K (tokens x key
        // dims), accumulated into the state registers
        const float c = c_s;
        const float wf[4] = {w_s[tg][jc], w_s[tg][jc + 1], w_s[tg + 4][jc], w_s[tg + 4][jc + 1]};
#pragma unroll
        for (int nb = 0; nb < 16; ++nb) {
            uint32_t bh0, bl0, bh1, bl1;
            split_tf32(k_s[tg][8 * nb + g], bh0, bl0);
            split_tf32(k_s[tg + 4][8 * nb + g], bh1, bl1);
#pragma unroll
            for (int i = 0; i < 4; ++i) s[nb][i] *= c;
            mma_f32_split<kExact>(s[nb], wf, bh0, bh1, bl0, bl1);
            float *p = st + (size_t)(8 * nb + 2 * tg) * D + jc;
            __stcs(reinterpret_cast<float2 *>(p), make_float2(s[nb][0], s[nb][2]));
            __stcs(reinterpret_cast<float2 *>(p + D), make_float2(s[nb][1], s[nb][3]));
        }

        __syncthreads();      // the shared arrays are reused by the next unit
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
    if (a.Dk == 128 && a.Dv == 128) {
        // one or two tokens: the paired-FMA kernel streams the state in 16-byte
        // pieces and is faster; from three tokens the products dominate
        if (a.T <= 2) return launch_shape<Tio, 128, 128>(a, s);
        static cudaError_t attr = cudaFuncSetAttribute(decode_tokens_tc_kernel<Tio>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)kTcSmem);
        if (attr != cudaSuccess) return attr;
        int dev = 0, sms = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        const long units = (long)a.B * a.H;
        const unsigned grid = (unsigned)(units < 2L * sms ? units : 2L * sms);   // two CTAs per SM
        decode_tokens_tc_kernel<Tio><<<grid, kThreads, kTcSmem, s>>>(a);
        return cudaGetLastError();
    }
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
