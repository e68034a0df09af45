// scan.cu -- the delta-rule recurrence, Eq.(2) of the review page of "Why
// Gated DeltaNet Survives 4-Bit Quantization" (paper sec.1):
//
//   S_t = alpha_t S_{t-1} + beta_t k_t (v_t - c_t S_{t-1}^T k_t)^T,   o_t = scale * S_t^T q_t
//
// with c_t = 1 (form PAGES, as the pages write it) or c_t = alpha_t (form
// STANDARD).  The state is float32 throughout.
//
// Two algorithms:
//  * recurrent: one CTA per (sequence, value head, 32-column slice of V); the
//    state slice lives in registers (thread = column, K/4 rows per warp), one
//    token per step.  Used for decode (T = 1) and as a reference path.
//  * chunked (C = 64 tokens): with G_t the running sum of g = log(alpha)
//    inside a chunk, the chunk's writes u solve the unit lower-triangular system
//      u_t + b_t sum_{i<t} e^{Gd_t - G_i} (k_t.k_i) u_i = beta_t v_t - b_t e^{Gd_t} S0^T k_t
//    (Gd_t = G_{t-1} for PAGES, G_t for STANDARD), i.e. U = U~ - W~ S0 with
//    U~ = T (beta V), W~ = T (D K), T = (I + L)^-1; then
//      o_t  = scale (e^{G_t} S0^T q_t + sum_{i<=t} e^{G_t - G_i} (q_t.k_i) u_i)
//      S_C  = e^{G_C} S0 + sum_i e^{G_C - G_i} k_i u_i^T.
//    Kernel 1 (parallel over chunk x head) builds W~, U~, the masked decayed
//    Q K^T and G; kernel 2 (one CTA per head x 32-column V slice) walks the
//    chunks in order.  Products run on the tensor cores in TF32 with float32
//    accumulation (mma.sync m16n8k8).
#include <cstdlib>
#include <cstring>

#include "common.cuh"

namespace nvg {

namespace {

constexpr int CH = 64;  // chunk length

// --------------------------------------------------------------- recurrent --
template <int K>
__global__ void __launch_bounds__(128) scan_recurrent_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v, int64_t ld_v,
    const float* __restrict__ g, const float* __restrict__ beta, int B, int64_t T, int Hk, int Hv, int V, float scale,
    int form, const float* state_in, float* state_out, float* __restrict__ o) {
    constexpr int RW = K / 4;
    const int nslice = V / 32;
    const int bh = blockIdx.x / nslice, slice = blockIdx.x - bh * nslice;
    const int b = bh / Hv, h = bh - b * Hv;
    const int hk = static_cast<int>((static_cast<int64_t>(h) * Hk) / Hv);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = slice * 32 + lane;
    const int64_t sbase = (static_cast<int64_t>(b) * Hv + h) * K * V;

    float S[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i) S[i] = state_in ? state_in[sbase + static_cast<int64_t>(w * RW + i) * V + j] : 0.0f;

    __shared__ float ks[K], qs[K];
    __shared__ float red1[4][32], red2[4][32];
    for (int64_t t = 0; t < T; ++t) {
        const int64_t tok = static_cast<int64_t>(b) * T + t;
        if (threadIdx.x < K) {
            ks[threadIdx.x] = k[(tok * Hk + hk) * K + threadIdx.x];
            qs[threadIdx.x] = q[(tok * Hk + hk) * K + threadIdx.x];
        }
        const float alpha = expf(g[tok * Hv + h]);
        const float bt = beta[tok * Hv + h];
        const float vj = v[tok * ld_v + static_cast<int64_t>(h) * V + j];
        __syncthreads();
        float p = 0.0f;
#pragma unroll
        for (int i = 0; i < RW; ++i) p = fmaf(S[i], ks[w * RW + i], p);
        red1[w][lane] = p;
        __syncthreads();
        float pred = (red1[0][lane] + red1[1][lane]) + (red1[2][lane] + red1[3][lane]);
        if (form == GDN_FORM_STANDARD) pred *= alpha;
        const float u = bt * (vj - pred);
        float acc = 0.0f;
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            S[i] = fmaf(alpha, S[i], ks[w * RW + i] * u);
            acc = fmaf(S[i], qs[w * RW + i], acc);
        }
        red2[w][lane] = acc;
        __syncthreads();
        if (w == 0) o[(tok * Hv + h) * V + j] = scale * ((red2[0][lane] + red2[1][lane]) + (red2[2][lane] + red2[3][lane]));
    }
    if (state_out) {
#pragma unroll
        for (int i = 0; i < RW; ++i) state_out[sbase + static_cast<int64_t>(w * RW + i) * V + j] = S[i];
    }
}

// ------------------------------------------------------------ mma helpers --
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// 3xTF32: a*b ~ a_hi b_hi + a_hi b_lo + a_lo b_hi (float32-level accuracy).
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = to_tf32(x);
    lo = to_tf32(x - __uint_as_float(hi));
}

template <bool PREC3>
__device__ __forceinline__ void mma_f32(float (&d)[4], const float (&a)[4], const float (&b)[2]) {
    if constexpr (PREC3) {
        uint32_t ah[4], al[4], bh[2], bl[2];
#pragma unroll
        for (int i = 0; i < 4; ++i) split_tf32(a[i], ah[i], al[i]);
        split_tf32(b[0], bh[0], bl[0]);
        split_tf32(b[1], bh[1], bl[1]);
        mma_tf32(d, al, bh);
        mma_tf32(d, ah, bl);
        mma_tf32(d, ah, bh);
    } else {
        const uint32_t ai[4] = {to_tf32(a[0]), to_tf32(a[1]), to_tf32(a[2]), to_tf32(a[3])};
        const uint32_t bi[2] = {to_tf32(b[0]), to_tf32(b[1])};
        mma_tf32(d, ai, bi);
    }
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------ chunk preparation --
// One CTA (256 threads) per (sequence, chunk, value head).
template <int K, int V>
struct PrepSmem {
    // row stride of the K and Q tiles (== 4 mod 32); the Q tile later holds the V rows
    static constexpr int KS = (K > V ? K : V) + 4;
    static constexpr int TS = CH + 4;  // row stride of T (== 4 mod 32)
    float ks[CH * KS];
    float qs[CH * KS];
    float L[CH * CH];                  // strictly lower, scaled: b_t e^{Gd_t - G_i} k_t.k_i
    float T[CH * TS];                  // (I + L)^-1
    float P[3 * 256];                  // 16 x 16 block products
    float gin[CH], gd[CH], bet[CH], graw[CH], df[CH];
};

// Output tile X [64 x 8*NT] = (T diag(s)) B with B [64 x 8*NT] (row stride KS) in
// shared memory; warp rows r0..r0+15; 3xTF32 (hi/lo split) so the product is
// float32-accurate.  X is written to global rows of `out` (row stride 8*NT),
// rounded to TF32 when `round_out`.
template <int NT, int KS, int TS>
__device__ __forceinline__ void tri_apply(const float* __restrict__ Tm, const float* __restrict__ s,
                                          const float* __restrict__ Bm, int r0, int lane, float* __restrict__ out,
                                          bool round_out) {
    const int grp = lane >> 2, tig = lane & 3;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll 2
    for (int k0 = 0; k0 < CH; k0 += 8) {
        const float s0 = s[k0 + tig], s1 = s[k0 + tig + 4];
        const float af[4] = {Tm[(r0 + grp) * TS + k0 + tig] * s0, Tm[(r0 + grp + 8) * TS + k0 + tig] * s0,
                             Tm[(r0 + grp) * TS + k0 + tig + 4] * s1, Tm[(r0 + grp + 8) * TS + k0 + tig + 4] * s1};
        uint32_t ah[4], al[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) split_tf32(af[i], ah[i], al[i]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            uint32_t bh[2], bl[2];
            split_tf32(Bm[(k0 + tig) * KS + nt * 8 + grp], bh[0], bl[0]);
            split_tf32(Bm[(k0 + tig + 4) * KS + nt * 8 + grp], bh[1], bl[1]);
            mma_tf32(acc[nt], al, bh);
            mma_tf32(acc[nt], ah, bl);
            mma_tf32(acc[nt], ah, bh);
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int t = r0 + grp + hh * 8;
            float x0 = acc[nt][2 * hh], x1 = acc[nt][2 * hh + 1];
            if (round_out) {
                x0 = __uint_as_float(to_tf32(x0));
                x1 = __uint_as_float(to_tf32(x1));
            }
            *reinterpret_cast<float2*>(out + t * (8 * NT) + nt * 8 + 2 * tig) = make_float2(x0, x1);
        }
    }
}

template <int K, int V>
__global__ void __launch_bounds__(256) chunk_prep_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                                         const float* __restrict__ v, int64_t ld_v,
                                                         const float* __restrict__ g, const float* __restrict__ beta,
                                                         int64_t T, int Hk, int Hv, int form, int NC,
                                                         float* __restrict__ Wt, float* __restrict__ Ut,
                                                         float* __restrict__ Mt, float* __restrict__ Gt) {
    using SM = PrepSmem<K, V>;
    constexpr int KS = SM::KS;
    extern __shared__ float4 smem_f4[];
    SM& sm = *reinterpret_cast<SM*>(smem_f4);
    const int h = blockIdx.x % Hv;
    const int c = (blockIdx.x / Hv) % NC;
    const int b = blockIdx.x / (Hv * NC);
    const int hk = static_cast<int>((static_cast<int64_t>(h) * Hk) / Hv);
    const int64_t t0 = static_cast<int64_t>(c) * CH;
    const int n = static_cast<int>((T - t0) < CH ? (T - t0) : CH);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // K, Q rows (zero past the end of the sequence) by asynchronous copies, g and beta
    constexpr int V4 = K / 4;
    for (int idx = tid; idx < CH * V4; idx += 256) {
        const int r = idx / V4, c4 = idx - r * V4;
        const bool valid = r < n;
        const int64_t off = valid ? ((static_cast<int64_t>(b) * T + t0 + r) * Hk + hk) * K + c4 * 4 : 0;
        cp_async16(&sm.ks[r * KS + c4 * 4], k + off, valid);
        cp_async16(&sm.qs[r * KS + c4 * 4], q + off, valid);
    }
    cp_async_commit();
    if (tid < CH) {
        const int64_t gi = (static_cast<int64_t>(b) * T + t0 + tid) * Hv + h;
        sm.graw[tid] = tid < n ? g[gi] : 0.0f;
        sm.bet[tid] = tid < n ? beta[gi] : 0.0f;
    }
    cp_async_wait<0>();
    __syncthreads();
    if (warp == 0) {
        // inclusive prefix sum of g over the chunk (2 values per lane)
        float a0 = sm.graw[2 * lane], a1 = sm.graw[2 * lane + 1];
        float s = a0 + a1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        const float excl = s - (a0 + a1);
        const float g0 = excl + a0, g1 = s;
        sm.gin[2 * lane] = g0;
        sm.gin[2 * lane + 1] = g1;
        sm.gd[2 * lane] = form == GDN_FORM_STANDARD ? g0 : excl;
        sm.gd[2 * lane + 1] = form == GDN_FORM_STANDARD ? g1 : g0;
    }
    __syncthreads();

    // K K^T (warps 0-3) and Q K^T (warps 4-7), 16 rows per warp, TF32 tensor cores
    {
        const int grp = lane >> 2, tig = lane & 3;
        const float* A = warp < 4 ? sm.ks : sm.qs;
        const int r0 = (warp & 3) * 16;
        float acc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll 4
        for (int k0 = 0; k0 < K; k0 += 8) {
            const float a[4] = {A[(r0 + grp) * KS + k0 + tig], A[(r0 + grp + 8) * KS + k0 + tig],
                                A[(r0 + grp) * KS + k0 + tig + 4], A[(r0 + grp + 8) * KS + k0 + tig + 4]};
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const float bb[2] = {sm.ks[(nt * 8 + grp) * KS + k0 + tig], sm.ks[(nt * 8 + grp) * KS + k0 + tig + 4]};
                mma_f32<false>(acc[nt], a, bb);
            }
        }
        const int64_t mbase = ((static_cast<int64_t>(b) * Hv + h) * NC + c) * CH * CH;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = r0 + grp + (e >> 1) * 8;
                const int i = nt * 8 + 2 * tig + (e & 1);
                if (warp < 4) {
                    sm.L[t * CH + i] = (i < t) ? sm.bet[t] * expf(sm.gd[t] - sm.gin[i]) * acc[nt][e] : 0.0f;
                } else {
                    // stored already rounded to TF32: it is only ever a tensor-core operand
                    const float mv = (i <= t) ? expf(sm.gin[t] - sm.gin[i]) * acc[nt][e] : 0.0f;
                    Mt[mbase + t * CH + i] = __uint_as_float(to_tf32(mv));
                }
            }
        }
    }
    if (tid < CH) {
        Gt[((static_cast<int64_t>(b) * Hv + h) * NC + c) * CH + tid] = sm.gin[tid];
        sm.df[tid] = sm.bet[tid] * expf(sm.gd[tid]);
    }
    constexpr int TS = SM::TS;
    for (int idx = tid; idx < CH * TS; idx += 256) sm.T[idx] = 0.0f;
    __syncthreads();
    // Q is no longer needed: its tile now receives the V rows (zero past the sequence
    // end); the copies land while the triangular inverse is formed
    constexpr int VV4 = V / 4;
    for (int idx = tid; idx < CH * VV4; idx += 256) {
        const int r = idx / VV4, c4 = idx - r * VV4;
        const bool valid = r < n;
        const int64_t off = valid ? (static_cast<int64_t>(b) * T + t0 + r) * ld_v + static_cast<int64_t>(h) * V + c4 * 4 : 0;
        cp_async16(&sm.qs[r * KS + c4 * 4], v + off, valid);
    }
    cp_async_commit();

    // T = (I + L)^-1, blockwise.  Diagonal 16 x 16 blocks by substitution
    // (warp w < 4 takes block w, lane c < 16 column c); then block rows
    // i = 1..3: T_ij = -T_ii sum_{k=j}^{i-1} L_ik T_kj.
    if (warp < 4 && lane < 16) {
        const int o = warp * 16;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = (r == lane) ? 1.0f : 0.0f;
#pragma unroll
            for (int i = 0; i < r; ++i) acc = fmaf(-sm.L[(o + r) * CH + o + i], x[i], acc);
            x[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) sm.T[(o + r) * TS + o + lane] = x[r];
    }
    __syncthreads();
    for (int bi = 1; bi < 4; ++bi) {
        for (int e = tid; e < bi * 256; e += 256) {
            const int j = e >> 8, r = (e >> 4) & 15, cc = e & 15;
            float acc = 0.0f;
            for (int kk = 16 * j; kk < 16 * bi; ++kk)
                acc = fmaf(sm.L[(16 * bi + r) * CH + kk], sm.T[kk * TS + 16 * j + cc], acc);
            sm.P[e] = acc;
        }
        __syncthreads();
        for (int e = tid; e < bi * 256; e += 256) {
            const int j = e >> 8, r = (e >> 4) & 15, cc = e & 15;
            float acc = 0.0f;
#pragma unroll
            for (int m = 0; m < 16; ++m) acc = fmaf(sm.T[(16 * bi + r) * TS + 16 * bi + m], sm.P[j * 256 + m * 16 + cc], acc);
            sm.T[(16 * bi + r) * TS + 16 * j + cc] = -acc;
        }
        __syncthreads();
    }

    cp_async_wait<0>();
    __syncthreads();
    // W~ = T diag(b e^{Gd}) K (warps 0-3, stored TF32-rounded: a tensor-core operand downstream)
    // U~ = T diag(beta) V   (warps 4-7)
    const int64_t cb = (static_cast<int64_t>(b) * Hv + h) * NC + c;
    if (warp < 4)
        tri_apply<K / 8, KS, TS>(sm.T, sm.df, sm.ks, warp * 16, lane, Wt + cb * CH * K, true);
    else
        tri_apply<V / 8, KS, TS>(sm.T, sm.bet, sm.qs, (warp - 4) * 16, lane, Ut + cb * CH * V, false);
}

// ------------------------------------------------------ sequential chunks --
template <int K>
struct SeqSmem {
    static constexpr int XS = K + 4;   // [W~; Q] tile row stride (== 4 mod 32)
    static constexpr int KS = K + 8;   // K tile row stride (== 8 mod 32, transposed reads)
    static constexpr int MS = CH + 4;  // masked Q K^T row stride
    static constexpr int SS = 40;      // state / U row stride (== 8 mod 32)
    float x1[2 * CH * XS];             // rows 0..63: W~ (TF32-rounded), rows 64..127: Q
    float kc[2][CH * KS];              // K of this chunk and the next one
    float mc[2][CH * MS];              // masked decayed Q K^T (TF32-rounded), double-buffered
    float s[K * SS];                   // float32 state slice [K x 32]
    float u[CH * SS];                  // U (TF32-rounded)
    float ud[CH * SS];                 // U scaled by e^{G_C - G_i} (TF32-rounded)
    float gin[2][CH];
};


// One CTA (256 threads) per (sequence, value head, 32-column slice of V).
// Per chunk: P1 = [W~; Q] S on all 8 warps (warps 0-3: W~ S, warps 4-7: Q S);
// warps 0-3 form U = U~ - W~ S; warps 4-7 then form o = scale (e^G Q S + M U)
// while every warp advances its 16 state rows S <- e^{G_C} S + K^T (decayed U).
// K, M and G of chunk c+1 are prefetched at the start of chunk c, W~ and Q of
// chunk c+1 as soon as P1 of chunk c has consumed them.
template <int K>
__global__ void __launch_bounds__(256) chunk_seq_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                                        int64_t T, int Hk, int Hv, int V, float scale, int NC,
                                                        const float* __restrict__ Wt, const float* __restrict__ Ut,
                                                        const float* __restrict__ Mt, const float* __restrict__ Gt,
                                                        const float* state_in, float* state_out, float* __restrict__ o) {
    using SM = SeqSmem<K>;
    constexpr int XS = SM::XS, KS = SM::KS, MS = SM::MS, SS = SM::SS;
    extern __shared__ float4 smem_f4[];
    SM& sm = *reinterpret_cast<SM*>(smem_f4);
    const int nslice = V / 32;
    const int slice = blockIdx.x % nslice;
    const int h = (blockIdx.x / nslice) % Hv;
    const int b = blockIdx.x / (nslice * Hv);
    const int hk = static_cast<int>((static_cast<int64_t>(h) * Hk) / Hv);
    const int vs0 = slice * 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = lane >> 2, tig = lane & 3;
    const int64_t sbase = (static_cast<int64_t>(b) * Hv + h) * K * V;
    const int64_t hc = (static_cast<int64_t>(b) * Hv + h) * NC;

    for (int idx = tid; idx < K * 32; idx += 256) {
        const int r = idx >> 5, cc = idx & 31;
        sm.s[r * SS + cc] = state_in ? state_in[sbase + static_cast<int64_t>(r) * V + vs0 + cc] : 0.0f;
    }

    auto load_wq = [&](int c) {
        const int64_t t0 = static_cast<int64_t>(c) * CH;
        constexpr int V4 = K / 4;
        for (int idx = tid; idx < CH * V4; idx += 256) {
            const int r = idx / V4, c4 = idx - r * V4;
            cp_async16(&sm.x1[r * XS + c4 * 4], Wt + ((hc + c) * CH + r) * K + c4 * 4, true);
            const bool valid = t0 + r < T;
            const int64_t qoff = valid ? ((static_cast<int64_t>(b) * T + t0 + r) * Hk + hk) * K + c4 * 4 : 0;
            cp_async16(&sm.x1[(CH + r) * XS + c4 * 4], q + qoff, valid);
        }
    };
    auto load_km = [&](int c, int buf) {
        const int64_t t0 = static_cast<int64_t>(c) * CH;
        constexpr int V4 = K / 4;
        for (int idx = tid; idx < CH * V4; idx += 256) {
            const int r = idx / V4, c4 = idx - r * V4;
            const bool valid = t0 + r < T;
            const int64_t koff = valid ? ((static_cast<int64_t>(b) * T + t0 + r) * Hk + hk) * K + c4 * 4 : 0;
            cp_async16(&sm.kc[buf][r * KS + c4 * 4], k + koff, valid);
        }
        for (int idx = tid; idx < CH * CH / 4; idx += 256) {
            const int r = idx >> 4, c4 = idx & 15;
            cp_async16(&sm.mc[buf][r * MS + c4 * 4], Mt + ((hc + c) * CH + r) * CH + c4 * 4, true);
        }
        if (tid < CH / 4) cp_async16(&sm.gin[buf][tid * 4], Gt + (hc + c) * CH + tid * 4, true);
    };

    load_wq(0);
    load_km(0, 0);
    cp_async_commit();

    for (int c = 0; c < NC; ++c) {
        const int64_t t0 = static_cast<int64_t>(c) * CH;
        const int buf = c & 1;
        cp_async_wait<0>();
        __syncthreads();
        if (c + 1 < NC) {
            load_km(c + 1, buf ^ 1);
            cp_async_commit();
        }
        // U~ for this warp's rows, fetched now so the latency hides behind P1
        float ut[4][4];
        if (warp < 4) {
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int i = warp * 16 + grp + hh * 8;
                    const float2 v2 = *reinterpret_cast<const float2*>(Ut + ((hc + c) * CH + i) * V + vs0 + nt * 8 + 2 * tig);
                    ut[nt][2 * hh] = v2.x;
                    ut[nt][2 * hh + 1] = v2.y;
                }
        }

        // P1: [W~; Q] (128 x K) times S (K x 32); warp w owns rows 16w..16w+15
        float acc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        {
            const int r0 = warp * 16;
            const bool a_rounded = warp < 4;  // W~ rows arrive rounded to TF32
#pragma unroll 4
            for (int k0 = 0; k0 < K; k0 += 8) {
                const float af[4] = {sm.x1[(r0 + grp) * XS + k0 + tig], sm.x1[(r0 + grp + 8) * XS + k0 + tig],
                                     sm.x1[(r0 + grp) * XS + k0 + tig + 4], sm.x1[(r0 + grp + 8) * XS + k0 + tig + 4]};
                uint32_t a[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = a_rounded ? __float_as_uint(af[i]) : to_tf32(af[i]);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const uint32_t bb[2] = {to_tf32(sm.s[(k0 + tig) * SS + nt * 8 + grp]),
                                            to_tf32(sm.s[(k0 + tig + 4) * SS + nt * 8 + grp])};
                    mma_tf32(acc[nt], a, bb);
                }
            }
        }
        const float glast = sm.gin[buf][CH - 1];
        if (warp < 4) {
            // U = U~ - W~ S0, and U decayed by e^{G_C - G_i} for the state update
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int i = warp * 16 + grp + hh * 8;
                const float dec = expf(glast - sm.gin[buf][i]);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                    for (int e1 = 0; e1 < 2; ++e1) {
                        const int e = 2 * hh + e1;
                        const int col = nt * 8 + 2 * tig + e1;
                        const float uval = ut[nt][e] - acc[nt][e];
                        sm.u[i * SS + col] = __uint_as_float(to_tf32(uval));
                        sm.ud[i * SS + col] = __uint_as_float(to_tf32(dec * uval));
                    }
                }
            }
        }
        __syncthreads();
        // X1 is free: prefetch the next chunk's W~ and Q while this chunk finishes
        if (c + 1 < NC) {
            load_wq(c + 1);
            cp_async_commit();
        }

        if (warp >= 4) {
            // o = scale * (e^{G_t} Q S0 + Mqk U); rows t = 16(w-4)..
            const int r0 = (warp - 4) * 16;
            const float* mc = sm.mc[buf];
            float mu[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) mu[nt][0] = mu[nt][1] = mu[nt][2] = mu[nt][3] = 0.f;
#pragma unroll
            for (int k0 = 0; k0 < CH; k0 += 8) {
                const uint32_t a[4] = {__float_as_uint(mc[(r0 + grp) * MS + k0 + tig]),
                                       __float_as_uint(mc[(r0 + grp + 8) * MS + k0 + tig]),
                                       __float_as_uint(mc[(r0 + grp) * MS + k0 + tig + 4]),
                                       __float_as_uint(mc[(r0 + grp + 8) * MS + k0 + tig + 4])};
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const uint32_t bb[2] = {__float_as_uint(sm.u[(k0 + tig) * SS + nt * 8 + grp]),
                                            __float_as_uint(sm.u[(k0 + tig + 4) * SS + nt * 8 + grp])};
                    mma_tf32(mu[nt], a, bb);
                }
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int t = r0 + grp + hh * 8;
                if (t0 + t < T) {
                    const float eg = expf(sm.gin[buf][t]);
                    float* orow = o + ((static_cast<int64_t>(b) * T + t0 + t) * Hv + h) * V + vs0;
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) {
                        const int col = nt * 8 + 2 * tig;
                        *reinterpret_cast<float2*>(orow + col) =
                            make_float2(scale * fmaf(eg, acc[nt][2 * hh], mu[nt][2 * hh]),
                                        scale * fmaf(eg, acc[nt][2 * hh + 1], mu[nt][2 * hh + 1]));
                    }
                }
            }
        }

        // S <- e^{G_C} S + K^T (diag(e^{G_C - G}) U); warp w owns state rows 16w..16w+15
        if (warp * 16 < K) {
            const int d0 = warp * 16;
            const float eg = expf(glast);
            const float* kc = sm.kc[buf];
            float st[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int col = nt * 8 + 2 * tig;
                st[nt][0] = eg * sm.s[(d0 + grp) * SS + col];
                st[nt][1] = eg * sm.s[(d0 + grp) * SS + col + 1];
                st[nt][2] = eg * sm.s[(d0 + grp + 8) * SS + col];
                st[nt][3] = eg * sm.s[(d0 + grp + 8) * SS + col + 1];
            }
#pragma unroll
            for (int k0 = 0; k0 < CH; k0 += 8) {
                const uint32_t a[4] = {to_tf32(kc[(k0 + tig) * KS + d0 + grp]), to_tf32(kc[(k0 + tig) * KS + d0 + grp + 8]),
                                       to_tf32(kc[(k0 + tig + 4) * KS + d0 + grp]),
                                       to_tf32(kc[(k0 + tig + 4) * KS + d0 + grp + 8])};
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const uint32_t bb[2] = {__float_as_uint(sm.ud[(k0 + tig) * SS + nt * 8 + grp]),
                                            __float_as_uint(sm.ud[(k0 + tig + 4) * SS + nt * 8 + grp])};
                    mma_tf32(st[nt], a, bb);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int col = nt * 8 + 2 * tig;
                sm.s[(d0 + grp) * SS + col] = st[nt][0];
                sm.s[(d0 + grp) * SS + col + 1] = st[nt][1];
                sm.s[(d0 + grp + 8) * SS + col] = st[nt][2];
                sm.s[(d0 + grp + 8) * SS + col + 1] = st[nt][3];
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();
    __syncthreads();
    if (state_out) {
        for (int idx = tid; idx < K * 32; idx += 256) {
            const int r = idx >> 5, cc = idx & 31;
            state_out[sbase + static_cast<int64_t>(r) * V + vs0 + cc] = sm.s[r * SS + cc];
        }
    }
}

// ------------------------------------------- sequential chunks, tcgen05 --
// Same per-chunk algebra as chunk_seq_kernel, on the sm_100 tensor cores: every
// product reads its operands from shared memory (no-swizzle K-major canonical
// tiles: 8-row x 16-byte core matrices) and accumulates in TMEM, so the warps
// only move data between the two MMA rounds of a chunk:
//   round 1:  D1 = [Q~; W~] S0            (M=128: rows 0..63 Q~ S0, 64..127 W~ S0)
//   warps 2-3: U = U~ - W~ S0, Ud = diag(e^{G_C - G}) U  -> shared memory
//   round 2:  D1 += [Mqk; *] U           (rows 0..63 become Q~ S0 + Mqk U;
//                                          the W~ S0 rows receive garbage, unused)
//             D2  = K^T Ud               (M=128 state rows)
//   warps 0-1: o = scale * D1[0:64];  all: S <- e^{G_C} S + D2 (float32 registers)
// Q~ = diag(e^{G}) Q is formed while rounding Q to TF32 in shared memory; K^T is
// built from the staged K tile in the same pass.
template <int K>
struct SeqTcSmem {
    static constexpr int A1_SBO = (K / 4) * 128;   // [Q~; W~] over the state dim: 8-row group stride
    static constexpr int T_SBO = 16 * 128;         // tiles whose K extent is the 64 tokens
    static constexpr int B1_SBO = (K / 4) * 128;   // S^T [32 x K]
    float a1[128 * K];
    float a2[2][64 * 64];                          // Mqk; a2[1] doubles as a2[0]'s unused upper rows
    float kst[2][64 * K];                          // staged K rows [t][d]; kst[0] follows a2[1]
    float a3[128 * 64];                            // K^T [d][t] (K = 64: upper half unused)
    float b1[32 * K];                              // S^T [v][d]
    float b2[32 * 64];                             // U^T [v][t]
    float b3[32 * 64];                             // Ud^T
    float gin[2][CH];
    uint64_t bar[2];
    uint32_t tmem_holder;
};

template <int K>
__global__ void __launch_bounds__(128) chunk_seq_tc_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                                           int64_t T, int Hk, int Hv, int V, float scale, int NC,
                                                           const float* __restrict__ Wt, const float* __restrict__ Ut,
                                                           const float* __restrict__ Mt, const float* __restrict__ Gt,
                                                           const float* state_in, float* state_out,
                                                           float* __restrict__ o, unsigned int* __restrict__ err) {
    using SM = SeqTcSmem<K>;
    extern __shared__ float4 smem_f4[];
    SM& sm = *reinterpret_cast<SM*>(smem_f4);
    const int nslice = V / 32;
    const int slice = blockIdx.x % nslice;
    const int h = (blockIdx.x / nslice) % Hv;
    const int b = blockIdx.x / (nslice * Hv);
    const int hk = static_cast<int>((static_cast<int64_t>(h) * Hk) / Hv);
    const int vs0 = slice * 32;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t sbase = (static_cast<int64_t>(b) * Hv + h) * K * V;
    const int64_t hc = (static_cast<int64_t>(b) * Hv + h) * NC;
    constexpr uint32_t IDESC = idesc_tf32(128, 32, false, false);

    if (tid == 0) {
        mbar_init(&sm.bar[0], 1);
        mbar_init(&sm.bar[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_holder, 64);
        tmem_relinquish();
    }

    // float offsets inside K-major canonical tiles: row r, column c, `cw` columns per row
    auto kmaj = [](int r, int c, int cw) { return ((r >> 3) * (cw >> 2) + (c >> 2)) * 32 + (r & 7) * 4 + (c & 3); };

    // state rows in registers: thread d < K holds S[d][vs0 .. vs0+31]
    float S[32];
    const bool has_row = tid < K;
    if (has_row) {
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (state_in) x = *reinterpret_cast<const float4*>(state_in + sbase + static_cast<int64_t>(tid) * V + vs0 + 4 * v4);
            S[4 * v4] = x.x; S[4 * v4 + 1] = x.y; S[4 * v4 + 2] = x.z; S[4 * v4 + 3] = x.w;
        }
#pragma unroll
        for (int v = 0; v < 32; ++v) sm.b1[kmaj(v, tid, K)] = __uint_as_float(to_tf32(S[v]));
    }

    auto load_wq = [&](int c) {
        const int64_t t0 = static_cast<int64_t>(c) * CH;
        for (int idx = tid; idx < CH * (K / 4); idx += 128) {
            const int t = idx / (K / 4), d4 = idx % (K / 4);
            cp_async16(&sm.a1[kmaj(CH + t, 4 * d4, K)], Wt + ((hc + c) * CH + t) * K + 4 * d4, true);
            const bool valid = t0 + t < T;
            const int64_t qoff = valid ? ((static_cast<int64_t>(b) * T + t0 + t) * Hk + hk) * K + 4 * d4 : 0;
            cp_async16(&sm.a1[kmaj(t, 4 * d4, K)], q + qoff, valid);
        }
    };
    auto load_kmg = [&](int c, int buf) {
        const int64_t t0 = static_cast<int64_t>(c) * CH;
        for (int idx = tid; idx < CH * (K / 4); idx += 128) {
            const int t = idx / (K / 4), d4 = idx % (K / 4);
            const bool valid = t0 + t < T;
            const int64_t koff = valid ? ((static_cast<int64_t>(b) * T + t0 + t) * Hk + hk) * K + 4 * d4 : 0;
            cp_async16(&sm.kst[buf][t * K + 4 * d4], k + koff, valid);
        }
        for (int idx = tid; idx < CH * 16; idx += 128) {
            const int t = idx >> 4, i4 = idx & 15;
            cp_async16(&sm.a2[buf][kmaj(t, 4 * i4, CH)], Mt + ((hc + c) * CH + t) * CH + 4 * i4, true);
        }
        if (tid < CH / 4) cp_async16(&sm.gin[buf][4 * tid], Gt + (hc + c) * CH + 4 * tid, true);
    };
    float ut[32];
    auto load_ut = [&](int c) {
        if (warp >= 2) {
            const float* src = Ut + ((hc + c) * CH + (tid - 64)) * V + vs0;
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4) {
                const float4 x = *reinterpret_cast<const float4*>(src + 4 * v4);
                ut[4 * v4] = x.x; ut[4 * v4 + 1] = x.y; ut[4 * v4 + 2] = x.z; ut[4 * v4 + 3] = x.w;
            }
        }
    };

    load_wq(0);
    load_kmg(0, 0);
    cp_async_commit();
    load_ut(0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_holder;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t D1 = tmem, D2 = tmem + 32;
    bool ok = true;

    for (int c = 0; c < NC && ok; ++c) {
        const int buf = c & 1;
        const int64_t t0 = static_cast<int64_t>(c) * CH;
        cp_async_wait<0>();
        __syncthreads();
        // Q~ = e^{G_t} Q rounded to TF32 in place; K^T [d][t] built from the staged rows, rounded
        for (int idx = tid; idx < CH * (K / 4); idx += 128) {
            const int t = idx / (K / 4), d4 = idx % (K / 4);
            float4* qp = reinterpret_cast<float4*>(&sm.a1[kmaj(t, 4 * d4, K)]);
            const float eg = expf(sm.gin[buf][t]);
            const float4 xq = *qp;
            *qp = make_float4(__uint_as_float(to_tf32(eg * xq.x)), __uint_as_float(to_tf32(eg * xq.y)),
                              __uint_as_float(to_tf32(eg * xq.z)), __uint_as_float(to_tf32(eg * xq.w)));
            const float4 xk = *reinterpret_cast<const float4*>(&sm.kst[buf][t * K + 4 * d4]);
            sm.a3[kmaj(4 * d4 + 0, t, CH)] = __uint_as_float(to_tf32(xk.x));
            sm.a3[kmaj(4 * d4 + 1, t, CH)] = __uint_as_float(to_tf32(xk.y));
            sm.a3[kmaj(4 * d4 + 2, t, CH)] = __uint_as_float(to_tf32(xk.z));
            sm.a3[kmaj(4 * d4 + 3, t, CH)] = __uint_as_float(to_tf32(xk.w));
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (c + 1 < NC) {
            load_kmg(c + 1, buf ^ 1);
            cp_async_commit();
        }
        const float glast = sm.gin[buf][CH - 1];

        // ---- round 1: D1 = [Q~; W~] S0
        if (tid == 0) {
            tc_fence_after();
            const uint32_t a1 = smem_u32(sm.a1), b1 = smem_u32(sm.b1);
#pragma unroll
            for (int j = 0; j < K / 8; ++j)
                mma_tf32_ss(D1, sdesc_noswz(a1 + j * 256, 128, SM::A1_SBO), sdesc_noswz(b1 + j * 256, 128, SM::B1_SBO),
                            IDESC, j > 0 ? 1u : 0u);
            mma_commit(&sm.bar[0]);
        }
        // every thread waits; the outcome is made block-uniform before warp-collective TMEM loads
        ok = __syncthreads_and(mbar_wait(&sm.bar[0], c & 1, err, kErrTimeoutMma) ? 1 : 0) != 0;
        tc_fence_after();
        if (warp >= 2 && ok) {
            // U = U~ - W~ S0 for token i (TMEM lanes 64..127), and the decayed copy
            const int i = tid - 64;
            uint32_t x[32];
            tmem_ld_32x32b_x32(D1 + lane_base, x);
            tmem_wait_ld();
            const float dec = expf(glast - sm.gin[buf][i]);
#pragma unroll
            for (int v = 0; v < 32; ++v) {
                const float u = ut[v] - __uint_as_float(x[v]);
                sm.b2[kmaj(v, i, CH)] = __uint_as_float(to_tf32(u));
                sm.b3[kmaj(v, i, CH)] = __uint_as_float(to_tf32(dec * u));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // the [Q~; W~] tile is consumed: fetch the next chunk's
        if (c + 1 < NC) {
            load_wq(c + 1);
            cp_async_commit();
        }

        // ---- round 2: D1[0:64] += Mqk U ; D2 = K^T Ud
        if (tid == 0) {
            tc_fence_after();
            const uint32_t a2 = smem_u32(sm.a2[buf]), a3 = smem_u32(sm.a3);
            const uint32_t b2 = smem_u32(sm.b2), b3 = smem_u32(sm.b3);
#pragma unroll
            for (int j = 0; j < CH / 8; ++j)
                mma_tf32_ss(D1, sdesc_noswz(a2 + j * 256, 128, SM::T_SBO), sdesc_noswz(b2 + j * 256, 128, SM::T_SBO),
                            IDESC, 1u);
#pragma unroll
            for (int j = 0; j < CH / 8; ++j)
                mma_tf32_ss(D2, sdesc_noswz(a3 + j * 256, 128, SM::T_SBO), sdesc_noswz(b3 + j * 256, 128, SM::T_SBO),
                            IDESC, j > 0 ? 1u : 0u);
            mma_commit(&sm.bar[1]);
        }
        ok = __syncthreads_and(mbar_wait(&sm.bar[1], c & 1, err, kErrTimeoutMma) ? 1 : 0) != 0;
        tc_fence_after();
        if (ok) {
            if (warp < 2) {
                const int t = tid;
                uint32_t x[32];
                tmem_ld_32x32b_x32(D1 + lane_base, x);
                tmem_wait_ld();
                if (t0 + t < T) {
                    float* orow = o + ((static_cast<int64_t>(b) * T + t0 + t) * Hv + h) * V + vs0;
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4)
                        *reinterpret_cast<float4*>(orow + 4 * v4) =
                            make_float4(scale * __uint_as_float(x[4 * v4]), scale * __uint_as_float(x[4 * v4 + 1]),
                                        scale * __uint_as_float(x[4 * v4 + 2]), scale * __uint_as_float(x[4 * v4 + 3]));
                }
            }
            uint32_t x[32];
            tmem_ld_32x32b_x32(D2 + lane_base, x);
            tmem_wait_ld();
            if (has_row) {
                const float eg = expf(glast);
#pragma unroll
                for (int v = 0; v < 32; ++v) {
                    S[v] = fmaf(eg, S[v], __uint_as_float(x[v]));
                    sm.b1[kmaj(v, tid, K)] = __uint_as_float(to_tf32(S[v]));
                }
            }
            if (c + 1 < NC) load_ut(c + 1);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }
    cp_async_wait<0>();
    if (state_out && has_row) {
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4)
            *reinterpret_cast<float4*>(state_out + sbase + static_cast<int64_t>(tid) * V + vs0 + 4 * v4) =
                make_float4(S[4 * v4], S[4 * v4 + 1], S[4 * v4 + 2], S[4 * v4 + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

struct ChunkWs {
    float *Wt, *Ut, *Mt, *Gt;
    size_t bytes;
};

ChunkWs chunk_ws(void* base, int B, int64_t T, const gdn_dims& d) {
    const int64_t NC = (T + CH - 1) / CH;
    const int64_t units = static_cast<int64_t>(B) * d.Hv * NC;
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t w = al(units * CH * d.K * 4), u = al(units * CH * d.V * 4), m = al(units * CH * CH * 4),
                 gg = al(units * CH * 4);
    ChunkWs ws;
    char* p = static_cast<char*>(base);
    ws.Wt = reinterpret_cast<float*>(p);
    ws.Ut = reinterpret_cast<float*>(p + w);
    ws.Mt = reinterpret_cast<float*>(p + w + u);
    ws.Gt = reinterpret_cast<float*>(p + w + u + m);
    ws.bytes = w + u + m + gg;
    return ws;
}

template <int K, int V>
nvfp4_status launch_chunked_kv(const float* q, const float* k, const float* v, int64_t ld_v, const float* g,
                               const float* beta, int B, int64_t T, const gdn_dims& d, float scale, int form,
                               const float* s_in, float* s_out, float* o, const ChunkWs& ws, cudaStream_t st) {
    const int NC = static_cast<int>((T + CH - 1) / CH);
    const int prep_smem = sizeof(PrepSmem<K, V>);
    const int seq_smem = sizeof(SeqSmem<K>);
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(chunk_prep_kernel<K, V>, cudaFuncAttributeMaxDynamicSharedMemorySize, prep_smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prep)");
        e = cudaFuncSetAttribute(chunk_seq_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, seq_smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(seq)");
        e = cudaFuncSetAttribute(chunk_seq_tc_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(sizeof(SeqTcSmem<K>)));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(seq tc)");
        attr_done[dev] = true;
    }
    const unsigned prep_blocks = static_cast<unsigned>(static_cast<int64_t>(B) * NC * d.Hv);
    chunk_prep_kernel<K, V><<<prep_blocks, 256, prep_smem, st>>>(q, k, v, ld_v, g, beta, T, d.Hk, d.Hv, form, NC, ws.Wt,
                                                                 ws.Ut, ws.Mt, ws.Gt);
    const unsigned seq_blocks = static_cast<unsigned>(B * d.Hv * (V / 32));
    const char* var = getenv("NVFP4_SCAN_SEQ_VARIANT");
    if (!var || strcmp(var, "tc") != 0) {
        chunk_seq_kernel<K><<<seq_blocks, 256, seq_smem, st>>>(q, k, T, d.Hk, d.Hv, V, scale, NC, ws.Wt, ws.Ut, ws.Mt,
                                                               ws.Gt, s_in, s_out, o);
    } else {
        unsigned int* err = device_error_word();
        if (!err) return fail(NVFP4_ERR_CUDA, "device error word unavailable");
        chunk_seq_tc_kernel<K><<<seq_blocks, 128, sizeof(SeqTcSmem<K>), st>>>(q, k, T, d.Hk, d.Hv, V, scale, NC, ws.Wt,
                                                                              ws.Ut, ws.Mt, ws.Gt, s_in, s_out, o, err);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "chunked scan launch");
    return NVFP4_OK;
}

}  // namespace

nvfp4_status validate_dims(const gdn_dims* d);

size_t scan_workspace_bytes(int B, int64_t T, const gdn_dims& d, int algo) {
    const bool chunked = algo == GDN_SCAN_CHUNKED || (algo == GDN_SCAN_AUTO && T > 1);
    if (!chunked) return 0;
    return chunk_ws(nullptr, B, T, d).bytes;
}

nvfp4_status scan_launch(const float* q, const float* k, const float* v, int64_t ld_v, const float* g,
                         const float* beta, int B, int64_t T, const gdn_dims& d, float scale, int form, int algo,
                         const float* s_in, float* s_out, float* o, void* ws, cudaStream_t st) {
    const bool chunked = algo == GDN_SCAN_CHUNKED || (algo == GDN_SCAN_AUTO && T > 1);
    if (!chunked) {
        const unsigned blocks = static_cast<unsigned>(B * d.Hv * (d.V / 32));
        if (d.K == 128)
            scan_recurrent_kernel<128><<<blocks, 128, 0, st>>>(q, k, v, ld_v, g, beta, B, T, d.Hk, d.Hv, d.V, scale, form,
                                                               s_in, s_out, o);
        else
            scan_recurrent_kernel<64><<<blocks, 128, 0, st>>>(q, k, v, ld_v, g, beta, B, T, d.Hk, d.Hv, d.V, scale, form,
                                                              s_in, s_out, o);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "recurrent scan launch");
        return NVFP4_OK;
    }
    const ChunkWs cws = chunk_ws(ws, B, T, d);
    if (d.K == 128 && d.V == 128)
        return launch_chunked_kv<128, 128>(q, k, v, ld_v, g, beta, B, T, d, scale, form, s_in, s_out, o, cws, st);
    if (d.K == 128 && d.V == 64)
        return launch_chunked_kv<128, 64>(q, k, v, ld_v, g, beta, B, T, d, scale, form, s_in, s_out, o, cws, st);
    if (d.K == 64 && d.V == 128)
        return launch_chunked_kv<64, 128>(q, k, v, ld_v, g, beta, B, T, d, scale, form, s_in, s_out, o, cws, st);
    return launch_chunked_kv<64, 64>(q, k, v, ld_v, g, beta, B, T, d, scale, form, s_in, s_out, o, cws, st);
}

}  // namespace nvg

extern "C" size_t gdn_scan_workspace_size(int32_t B, int64_t T, const gdn_dims* dims, int32_t algo) {
    if (!dims || nvg::validate_dims(dims) != NVFP4_OK || B < 1 || T < 1) return 0;
    return nvg::scan_workspace_bytes(B, T, *dims, algo);
}

extern "C" nvfp4_status gdn_scan(const float* q_hat, const float* k_hat, const float* v, int64_t ld_v, const float* g,
                                 const float* beta, int32_t B, int64_t T, const gdn_dims* dims, float scale,
                                 int32_t form, int32_t algo, const float* state_in, float* state_out, float* o,
                                 void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
    using namespace nvg;
    nvfp4_status s = validate_dims(dims);
    if (s != NVFP4_OK) return s;
    if (!q_hat || !k_hat || !v || !g || !beta || !o) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
    if (B < 1 || T < 1) return fail(NVFP4_ERR_INVALID_ARG, "B and T must be >= 1");
    if (form != GDN_FORM_PAGES && form != GDN_FORM_STANDARD) return fail(NVFP4_ERR_INVALID_ARG, "bad form");
    if (algo != GDN_SCAN_AUTO && algo != GDN_SCAN_RECURRENT && algo != GDN_SCAN_CHUNKED)
        return fail(NVFP4_ERR_INVALID_ARG, "bad algo");
    if (ld_v < static_cast<int64_t>(dims->Hv) * dims->V) return fail(NVFP4_ERR_INVALID_ARG, "ld_v < Hv*V");
    if (static_cast<int64_t>(B) * T > (int64_t(1) << 31)) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "B*T too large");
    if (!aligned16(q_hat) || !aligned16(k_hat) || !aligned16(o) || !aligned16(v) || ld_v % 4)
        return fail(NVFP4_ERR_MISALIGNED, "q_hat, k_hat, v, o must be 16-byte aligned and ld_v % 4 == 0");
    const size_t need = scan_workspace_bytes(B, T, *dims, algo);
    if (need && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255)))
        return fail(NVFP4_ERR_WORKSPACE, "scan workspace missing, too small or not 256-byte aligned");
    return scan_launch(q_hat, k_hat, v, ld_v, g, beta, B, T, *dims, scale, form, algo, state_in, state_out, o,
                       workspace, as_stream(stream));
}
