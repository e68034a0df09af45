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
#include <algorithm>
#include <type_traits>

#include "common.cuh"

namespace nvg {

nvfp4_status identity_fill_launch(float* P, int64_t n_mat, int K, float* zero_row, int64_t n_zero, cudaStream_t st);
size_t transition_workspace_bytes(int B, int64_t T, const gdn_dims& d, int algo);

namespace {

constexpr int CH = 64;  // chunk length

// Byte offset of element (r, col) in a K-major tcgen05 operand image with the
// 128-byte swizzle: the columns are split into 32-float atom columns, each
// holding `rows` rows of 128 bytes; inside an 8-row group the 16-byte chunk
// index is XORed with the row index (r mod 8).  Atom columns start on 1024-byte
// boundaries.
__host__ __device__ constexpr uint32_t sw128_off(int r, int col, int rows) {
    return static_cast<uint32_t>((col >> 5) * rows * 128 + r * 128 + ((((col & 31) >> 2) ^ (r & 7)) << 4) +
                                 ((col & 3) << 2));
}

// Per (sequence, value head, chunk) record written by the preparation kernel
// and copied, section by section, into the sequential kernel's shared memory:
//   A1  [Q~; W~]  128 x K   Q~ = diag(e^{G}) Q (rows 0..63), W~ (rows 64..127)
//   A2  Mqk       64 x 64   masked decayed Q K^T, M_ti = e^{G_t - G_i} q_t.k_i (i <= t)
//   A3  K^ ^T     K x 64    K^_t = e^{G_C - G_t} k_t (atom columns of 128 rows)
//   UT  U~        64 x V    one 8 KB swizzled 64 x 32 tile per 32-column slice
//   GC  G_C       the chunk's total log-decay
// A1..A3 hold TF32-rounded values in the swizzled layout above; U~ is float32.
template <int K, int V>
struct ChunkRec {
    static constexpr uint32_t A1 = 0;
    static constexpr uint32_t A1_BYTES = 128 * K * 4;
    static constexpr uint32_t A2 = A1 + A1_BYTES;
    static constexpr uint32_t A2_BYTES = CH * CH * 4;
    static constexpr uint32_t A3 = A2 + A2_BYTES;
    static constexpr uint32_t A3_BYTES = 2 * 128 * 128;
    static constexpr uint32_t UT = A3 + A3_BYTES;
    static constexpr uint32_t UT_SLICE = CH * 32 * 4;
    static constexpr uint32_t GC = UT + (V / 32) * UT_SLICE;
    static constexpr uint32_t BYTES = GC + 1024;
};

// --------------------------------------------------------------- recurrent --
// q and k rows of token (b, t) at (b*T + t) * ld_qk (+ key head * K); with
// normalize_qk they are the raw projection slices and are scaled here by
// 1 / sqrt(sum x^2 + 1e-6) per key head.
template <int K>
__global__ void __launch_bounds__(128) scan_recurrent_kernel(
    const float* __restrict__ q, const float* __restrict__ k, int64_t ld_qk, int normalize_qk,
    const float* __restrict__ v, int64_t ld_v,
    const float* __restrict__ g, const float* __restrict__ beta, int B, int64_t T, int Hk, int Hv, int V, float scale,
    int form, const float* state_in, float* state_out, float* __restrict__ o, unsigned int* __restrict__ o_amax) {
    pdl_wait_and_trigger();
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
    __shared__ float inv_norm[2];
    for (int64_t t = 0; t < T; ++t) {
        const int64_t tok = static_cast<int64_t>(b) * T + t;
        if (threadIdx.x < K) {
            ks[threadIdx.x] = k[tok * ld_qk + static_cast<int64_t>(hk) * K + threadIdx.x];
            qs[threadIdx.x] = q[tok * ld_qk + static_cast<int64_t>(hk) * K + threadIdx.x];
        }
        const float alpha = expf(g[tok * Hv + h]);
        const float bt = beta[tok * Hv + h];
        const float vj = v[tok * ld_v + static_cast<int64_t>(h) * V + j];
        __syncthreads();
        if (normalize_qk) {   // warp 0 takes |k|, warp 1 |q|
            if (w < 2) {
                const float* src = w == 0 ? ks : qs;
                float ss = 0.0f;
#pragma unroll
                for (int i = lane; i < K; i += 32) ss = fmaf(src[i], src[i], ss);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                if (lane == 0) inv_norm[w] = rsqrtf(ss + 1e-6f);
            }
            __syncthreads();
            if (threadIdx.x < K) {
                ks[threadIdx.x] *= inv_norm[0];
                qs[threadIdx.x] *= inv_norm[1];
            }
            __syncthreads();
        }
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
        if (w == 0) {
            const float ov = scale * ((red2[0][lane] + red2[1][lane]) + (red2[2][lane] + red2[3][lane]));
            o[(tok * Hv + h) * V + j] = ov;
            if (o_amax) {
                const unsigned int mb = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(ov)));
                if (lane == 0) atomicMax(o_amax, mb);
            }
        }
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

// Four 8 x 4 float32 matrices from shared memory, one 16-byte row address per
// lane (lanes 8i..8i+7 give the rows of matrix i).  Register i of lane l then
// holds element (l / 4, l % 4) of matrix i: with the matrices chosen as below this
// is a TF32 m16n8k8 A fragment (rows +0..7 | +8..15 x columns +0..3 | +4..7), or
// the B fragments of two 8-column tiles.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const float* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

// ------------------------------------------------------ chunk preparation --
// One CTA (256 threads) per (sequence, chunk, value head).
template <int K, int V>
struct PrepSmem {
    // row stride of the K and Q tiles (a multiple of 32 floats; the columns are
    // XOR-swizzled, see tile_off); the Q tile later holds the V rows
    static constexpr int KS = (K > V ? K : V);
    static constexpr int LS = CH + 4;  // row stride of L (== 4 mod 32)
    static constexpr int TBS = 20;     // row stride of the diagonal-block inverses
    float ks[CH * KS];
    float qs[CH * KS];
    float L[CH * LS];                  // -L (TF32): L strictly lower, L_ti = b_t e^{Gd_t - G_i} k_t.k_i
    float Tb[4 * 16 * TBS];            // (I + L_bb)^-1 for the four 16 x 16 diagonal blocks
    float gin[CH], gd[CH], bet[CH], graw[CH], df[CH];
    float eG[CH], eKh[CH];             // e^{G_t}, e^{G_C - G_t}
};

// W = (I + L)^-1 diag(s) X for the 32-column strip c0..c0+31 of X [64 x N] (row
// stride KS) in shared memory, by block forward substitution over 16-row blocks:
//   W_b = T_bb (diag(s_b) X_b - sum_{k<b} L_bk W_k),   T_bb = (I + L_bb)^-1.
// Lm holds -L and Tb the T_bb, X the right-hand sides, all already rounded to TF32;
// the strip is overwritten by W rounded to TF32 (it is only read again as an MMA
// operand) and each pair of adjacent float32 outputs (t, col), (t, col+1), col even,
// goes to store(t, col, x0, x1).  One warp, which alone touches these columns.
// TF32 tensor cores, float32 accumulation.
// Float offset of element (r, c) of a K, Q or V tile with row stride KS (a
// multiple of 32).  Bits 2..4 of the column are XORed with ((r & 3) << 3) | (r & 4),
// which permutes the 4-float groups inside each 32-float segment of a row.  Every
// access pattern of the tiles is then free of bank conflicts: the ldmatrix reads of
// TF32 mma.sync fragments with k along a row (eight 16-byte row pieces of eight
// consecutive rows), the B fragments read with k down the columns (rows tig,
// columns grp), the float2 accumulator accesses, and row-contiguous vector
// accesses.  Aligned 2- and 4-float vectors stay contiguous.
template <int KS>
__device__ __forceinline__ int tile_off(int r, int c) {
    static_assert(KS % 32 == 0, "tile stride must be a multiple of 32 floats");
    return r * KS + (c ^ (((r & 3) << 3) | (r & 4)));
}

template <int KS, int LS, int TBS, typename Store>
__device__ __forceinline__ void block_subst(const float* __restrict__ Lm, const float* __restrict__ Tb,
                                            const float* __restrict__ s, float* __restrict__ X, int c0, int lane,
                                            Store store) {
    const int grp = lane >> 2, tig = lane & 3;
    // row and column of this lane's ldmatrix address inside a 16 x 8 A fragment
    const int fr = (lane & 7) + ((lane >> 3) & 1) * 8, fc = (lane >> 4) * 4;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const int r0 = 16 * b;
        float acc[4][4];
        const float s0 = s[r0 + grp], s1 = s[r0 + grp + 8];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int col = c0 + nt * 8 + 2 * tig;
            const float2 x0 = *reinterpret_cast<const float2*>(&X[tile_off<KS>(r0 + grp, col)]);
            const float2 x1 = *reinterpret_cast<const float2*>(&X[tile_off<KS>(r0 + grp + 8, col)]);
            acc[nt][0] = s0 * x0.x;
            acc[nt][1] = s0 * x0.y;
            acc[nt][2] = s1 * x1.x;
            acc[nt][3] = s1 * x1.y;
        }
#pragma unroll
        for (int k0 = 0; k0 < r0; k0 += 8) {
            uint32_t a[4];
            ldsm_x4(a, &Lm[(r0 + fr) * LS + k0 + fc]);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const uint32_t bb[2] = {__float_as_uint(X[tile_off<KS>(k0 + tig, c0 + nt * 8 + grp)]),
                                        __float_as_uint(X[tile_off<KS>(k0 + tig + 4, c0 + nt * 8 + grp)])};
                mma_tf32(acc[nt], a, bb);
            }
        }
        // Y_b over X_b: every lane rewrites exactly the positions it read
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int col = c0 + nt * 8 + 2 * tig;
            *reinterpret_cast<float2*>(&X[tile_off<KS>(r0 + grp, col)]) =
                make_float2(__uint_as_float(to_tf32(acc[nt][0])), __uint_as_float(to_tf32(acc[nt][1])));
            *reinterpret_cast<float2*>(&X[tile_off<KS>(r0 + grp + 8, col)]) =
                make_float2(__uint_as_float(to_tf32(acc[nt][2])), __uint_as_float(to_tf32(acc[nt][3])));
        }
        __syncwarp();
        float w[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) w[nt][0] = w[nt][1] = w[nt][2] = w[nt][3] = 0.f;
        const float* Tbb = Tb + b * 16 * TBS;
#pragma unroll
        for (int k0 = 0; k0 < 16; k0 += 8) {
            uint32_t a[4];
            ldsm_x4(a, &Tbb[fr * TBS + k0 + fc]);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const uint32_t bb[2] = {__float_as_uint(X[tile_off<KS>(r0 + k0 + tig, c0 + nt * 8 + grp)]),
                                        __float_as_uint(X[tile_off<KS>(r0 + k0 + tig + 4, c0 + nt * 8 + grp)])};
                mma_tf32(w[nt], a, bb);
            }
        }
        __syncwarp();
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int col = c0 + nt * 8 + 2 * tig;
            *reinterpret_cast<float2*>(&X[tile_off<KS>(r0 + grp, col)]) =
                make_float2(__uint_as_float(to_tf32(w[nt][0])), __uint_as_float(to_tf32(w[nt][1])));
            *reinterpret_cast<float2*>(&X[tile_off<KS>(r0 + grp + 8, col)]) =
                make_float2(__uint_as_float(to_tf32(w[nt][2])), __uint_as_float(to_tf32(w[nt][3])));
            store(r0 + grp, col, w[nt][0], w[nt][1]);
            store(r0 + grp + 8, col, w[nt][2], w[nt][3]);
        }
        __syncwarp();
    }
}

template <int K, int V>
__global__ void __launch_bounds__(256) chunk_prep_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                                         int64_t ld_qk, int normalize_qk,
                                                         const float* __restrict__ v, int64_t ld_v,
                                                         const float* __restrict__ g, const float* __restrict__ beta,
                                                         int64_t T, int Hk, int Hv, int form, int NC,
                                                         uint8_t* __restrict__ recs) {
    pdl_wait_and_trigger();
    using SM = PrepSmem<K, V>;
    using RC = ChunkRec<K, V>;
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
    uint8_t* rec = recs + ((static_cast<int64_t>(b) * Hv + h) * NC + c) * RC::BYTES;

    // K, Q rows (zero past the end of the sequence) by asynchronous copies, g and beta;
    // token t's head hk row starts at (b T + t) ld_qk + hk K
    {
        // each thread copies one 16-byte column piece of every RS-th row
        constexpr int V4 = K / 4, RS = 256 / V4;
        const int c4 = tid % V4, r0 = tid / V4;
        const int64_t step = static_cast<int64_t>(RS) * ld_qk;
        int64_t off = (static_cast<int64_t>(b) * T + t0 + r0) * ld_qk + static_cast<int64_t>(hk) * K + c4 * 4;
#pragma unroll
        for (int r = r0; r < CH; r += RS, off += step) {
            const bool valid = r < n;
            const int so = tile_off<KS>(r, c4 * 4);
            cp_async16(&sm.ks[so], k + (valid ? off : 0), valid);
            cp_async16(&sm.qs[so], q + (valid ? off : 0), valid);
        }
    }
    cp_async_commit();
    if (tid < CH) {
        const int64_t gi = (static_cast<int64_t>(b) * T + t0 + tid) * Hv + h;
        sm.graw[tid] = tid < n ? g[gi] : 0.0f;
        sm.bet[tid] = tid < n ? beta[gi] : 0.0f;
    }
    cp_async_wait<0>();
    __syncthreads();
    {
        // K and Q tiles are tensor-core operands only from here on: rounded to TF32
        // in place.  With raw q, k rows (normalize_qk) each row is first scaled by
        // 1 / sqrt(sum x^2 + 1e-6), one warp per row, each lane K/32 contiguous values
        // (the same operation order as the standalone normalisation).
        // (Each lane moves its K/32 values as one vector access, so a warp's row is
        // contiguous in shared memory: no bank conflicts.)
        constexpr int PL = K / 32;
        static_assert(PL == 2 || PL == 4, "K must be 64 or 128");
        using VecT = typename std::conditional<PL == 4, float4, float2>::type;
        for (int row = warp; row < 2 * CH; row += 8) {
            VecT* x = reinterpret_cast<VecT*>((row < CH ? sm.ks : sm.qs) + tile_off<KS>(row % CH, lane * PL));
            const VecT xv = *x;
            float vv[PL];
            memcpy(vv, &xv, sizeof(vv));
            float inv = 1.0f;
            if (normalize_qk) {
                float ss = 0.0f;
#pragma unroll
                for (int i = 0; i < PL; ++i) ss = fmaf(vv[i], vv[i], ss);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                inv = rsqrtf(ss + 1e-6f);
            }
#pragma unroll
            for (int i = 0; i < PL; ++i) vv[i] = __uint_as_float(to_tf32(normalize_qk ? vv[i] * inv : vv[i]));
            VecT yv;
            memcpy(&yv, vv, sizeof(vv));
            *x = yv;
        }
        __syncthreads();
    }
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
        const float d0 = form == GDN_FORM_STANDARD ? g0 : excl;
        const float d1 = form == GDN_FORM_STANDARD ? g1 : g0;
        sm.gd[2 * lane] = d0;
        sm.gd[2 * lane + 1] = d1;
        const float gc = __shfl_sync(0xffffffffu, g1, 31);
        sm.eG[2 * lane] = expf(g0);
        sm.eG[2 * lane + 1] = expf(g1);
        sm.eKh[2 * lane] = expf(gc - g0);
        sm.eKh[2 * lane + 1] = expf(gc - g1);
        sm.df[2 * lane] = sm.bet[2 * lane] * expf(d0);
        sm.df[2 * lane + 1] = sm.bet[2 * lane + 1] * expf(d1);
    }
    __syncthreads();

    // K K^T (warps 0-3) and Q K^T (warps 4-7), 16 rows per warp, TF32 tensor cores
    {
        const int grp = lane >> 2, tig = lane & 3;
        const float* A = warp < 4 ? sm.ks : sm.qs;
        const int r0 = (warp & 3) * 16;
        // tiles right of this warp's diagonal block are skipped (masked out afterwards):
        // it takes 8-column tiles 0 .. r0/8 + 1, two per B load
        const int npairs = (r0 >> 4) + 1;
        // ldmatrix addresses: A rows r0 + ar, columns + ac; B rows 16 np + br, columns + bc
        const int ar = r0 + (lane & 7) + ((lane >> 3) & 1) * 8, ac = (lane >> 4) * 4;
        const int br = (lane & 7) + (lane >> 4) * 8, bc = ((lane >> 3) & 1) * 4;
        float acc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll 4
        for (int k0 = 0; k0 < K; k0 += 8) {
            uint32_t ai[4];
            ldsm_x4(ai, &A[tile_off<KS>(ar, k0 + ac)]);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                if (np >= npairs) continue;
                uint32_t bq[4];
                ldsm_x4(bq, &sm.ks[tile_off<KS>(16 * np + br, k0 + bc)]);
                const uint32_t b0[2] = {bq[0], bq[1]}, b1[2] = {bq[2], bq[3]};
                mma_tf32(acc[2 * np], ai, b0);
                mma_tf32(acc[2 * np + 1], ai, b1);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int t = r0 + grp + hh * 8;
                const int i = nt * 8 + 2 * tig;
                if (warp < 4) {
                    // stored negated and rounded to TF32: -L is a tensor-core operand
                    const float l0 = (i < t) ? sm.bet[t] * __expf(sm.gd[t] - sm.gin[i]) * acc[nt][2 * hh] : 0.0f;
                    const float l1 =
                        (i + 1 < t) ? sm.bet[t] * __expf(sm.gd[t] - sm.gin[i + 1]) * acc[nt][2 * hh + 1] : 0.0f;
                    *reinterpret_cast<float2*>(&sm.L[t * SM::LS + i]) =
                        make_float2(__uint_as_float(to_tf32(-l0)), __uint_as_float(to_tf32(-l1)));
                } else {
                    // rounded to TF32 here: it is only ever a tensor-core operand
                    const float m0 = (i <= t) ? __expf(sm.gin[t] - sm.gin[i]) * acc[nt][2 * hh] : 0.0f;
                    const float m1 = (i + 1 <= t) ? __expf(sm.gin[t] - sm.gin[i + 1]) * acc[nt][2 * hh + 1] : 0.0f;
                    *reinterpret_cast<float2*>(rec + RC::A2 + sw128_off(t, i, CH)) =
                        make_float2(__uint_as_float(to_tf32(m0)), __uint_as_float(to_tf32(m1)));
                }
            }
        }
    }
    if (tid == 0) *reinterpret_cast<float*>(rec + RC::GC) = sm.gin[CH - 1];
    // Q~ = e^{G_t} q_t (rows 0..63 of A1) and K^ ^T, K^_t = e^{G_C - G_t} k_t (A3), TF32-rounded
    for (int idx = tid; idx < CH * (K / 4); idx += 256) {
        const int t = idx / (K / 4), c4 = idx - t * (K / 4);
        const float eg = sm.eG[t];
        const float4 x = *reinterpret_cast<const float4*>(&sm.qs[tile_off<KS>(t, 4 * c4)]);
        *reinterpret_cast<float4*>(rec + RC::A1 + sw128_off(t, 4 * c4, 128)) =
            make_float4(__uint_as_float(to_tf32(eg * x.x)), __uint_as_float(to_tf32(eg * x.y)),
                        __uint_as_float(to_tf32(eg * x.z)), __uint_as_float(to_tf32(eg * x.w)));
    }
    for (int idx = tid; idx < K * (CH / 4); idx += 256) {
        const int dd = idx % K, t4 = idx / K;
        float x[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) x[w] = __uint_as_float(to_tf32(sm.eKh[4 * t4 + w] * sm.ks[tile_off<KS>(4 * t4 + w, dd)]));
        *reinterpret_cast<float4*>(rec + RC::A3 + sw128_off(dd, 4 * t4, 128)) = make_float4(x[0], x[1], x[2], x[3]);
    }
    __syncthreads();
    // Q is no longer needed: its tile now receives the V rows (zero past the sequence
    // end); the copies land while the diagonal blocks are inverted
    {
        constexpr int VV4 = V / 4, RS = 256 / VV4;
        const int c4 = tid % VV4, r0 = tid / VV4;
        const int64_t step = static_cast<int64_t>(RS) * ld_v;
        int64_t off = (static_cast<int64_t>(b) * T + t0 + r0) * ld_v + static_cast<int64_t>(h) * V + c4 * 4;
#pragma unroll
        for (int r = r0; r < CH; r += RS, off += step) {
            const bool valid = r < n;
            cp_async16(&sm.qs[tile_off<KS>(r, c4 * 4)], v + (valid ? off : 0), valid);
        }
    }
    cp_async_commit();

    // T_bb = (I + L_bb)^-1 for the four 16 x 16 diagonal blocks, by forward substitution
    // in registers: warp b takes block b, lane r (and r + 16) holds row r; once row i is
    // final it is broadcast and every later row r subtracts L_ri times it.
    constexpr int LS = SM::LS, TBS = SM::TBS;
    if (warp < 4) {
        const int o = 16 * warp, r = lane & 15;
        float Lr[16], Tr[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            Lr[i] = i < r ? sm.L[(o + r) * LS + o + i] : 0.0f;
            Tr[i] = i == r ? 1.0f : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < 15; ++i) {
#pragma unroll
            for (int j = 0; j <= i; ++j) {
                const float tij = __shfl_sync(0xffffffffu, Tr[j], i);
                Tr[j] = fmaf(Lr[i], tij, Tr[j]);   // Lr holds -L
            }
        }
        if (lane < 16) {
#pragma unroll
            for (int j = 0; j < 16; ++j) sm.Tb[warp * 16 * TBS + r * TBS + j] = __uint_as_float(to_tf32(Tr[j]));
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    for (int idx = tid; idx < CH * (V / 4); idx += 256) {
        float4* p4 = reinterpret_cast<float4*>(&sm.qs[tile_off<KS>(idx / (V / 4), 4 * (idx % (V / 4)))]);
        const float4 x = *p4;
        *p4 = make_float4(__uint_as_float(to_tf32(x.x)), __uint_as_float(to_tf32(x.y)), __uint_as_float(to_tf32(x.z)),
                          __uint_as_float(to_tf32(x.w)));
    }
    __syncthreads();
    // W~ = (I + L)^-1 diag(b e^{Gd}) K (stored TF32-rounded: a tensor-core operand downstream),
    // U~ = (I + L)^-1 diag(beta) V; 32-column strips, W~ strips first, one warp each
    for (int strip = warp; strip < K / 32 + V / 32; strip += 8) {
        if (strip < K / 32) {
            block_subst<KS, LS, TBS>(sm.L, sm.Tb, sm.df, sm.ks, 32 * strip, lane, [&](int t, int col, float x0, float x1) {
                *reinterpret_cast<float2*>(rec + RC::A1 + sw128_off(CH + t, col, 128)) =
                    make_float2(__uint_as_float(to_tf32(x0)), __uint_as_float(to_tf32(x1)));
            });
        } else {
            const int vs = strip - K / 32;
            block_subst<KS, LS, TBS>(sm.L, sm.Tb, sm.bet, sm.qs, 32 * vs, lane, [&](int t, int col, float x0, float x1) {
                *reinterpret_cast<float2*>(rec + RC::UT + vs * RC::UT_SLICE + sw128_off(t, col - 32 * vs, CH)) =
                    make_float2(x0, x1);
            });
        }
    }
}

// ------------------------------------------------------ sequential chunks --
// One CTA per (sequence, value head, 32-column slice of V) walks the chunks in
// order, on the tcgen05 tensor cores (kind::tf32, float32 accumulation in TMEM,
// M = 128, N = 32).  Per chunk:
//   R1:   D1 = [Q~; W~] S0          rows 0..63: Q~ S0, rows 64..127: W~ S0
//   U = U~ - W~ S0 (TF32)  ->  U^T in shared memory
//   R2a:  D2  = K^ ^T U              K^_t = e^{G_C - G_t} k_t
//   R2b:  D1 += [Mqk; *] U           rows 0..63: o / scale (rows 64..127 unused)
//   S <- e^{G_C} S + D2 (float32, registers)  ->  S^T (TF32) in shared memory
// The recurrence runs through R1 -> U -> R2a -> S only; R2b and the output rows
// drain while the next chunk's R1 and U run (D1 alternates between two TMEM
// buffers).  Warp 0 copies the chunk records into shared memory (bulk copies,
// [Q~; W~] and U~ double-buffered, L2 prefetch ahead) and issues R2b once R2a has
// completed; warp 1 issues R1 and R2a; the compute warps, kSeqGroups per TMEM lane
// quarter with kSeqCols columns each, form U, the state and the output.  Every
// hand-off is an mbarrier (bounded waits).
template <int K>
struct SeqLayout {
    static constexpr uint32_t A1_BYTES = 128 * K * 4;
    static constexpr uint32_t A1 = 0;                         // two stages
    static constexpr uint32_t A23 = 2 * A1_BYTES;             // Mqk (16 KB) then K^ ^T (32 KB)
    static constexpr uint32_t A23_BYTES = CH * CH * 4 + 2 * 128 * 128;
    static constexpr uint32_t UT = A23 + A23_BYTES;           // two stages of a 64 x 32 U~ slice
    static constexpr uint32_t UT_BYTES = CH * 32 * 4;
    static constexpr uint32_t B1 = UT + 2 * UT_BYTES;         // S^T: K/32 atom columns of 32 rows
    static constexpr uint32_t B2 = B1 + K * 128;              // U^T: 2 atom columns of 32 rows
    static constexpr uint32_t BAR = B2 + CH * 128;
    static constexpr uint32_t BYTES = BAR + 256 + 1024;       // + alignment slack
};

// warp 0: producer, warp 1: MMA, then kSeqGroups groups of 4 compute warps (one per
// TMEM lane quarter), group j owning columns 32 / kSeqGroups * j .. of the slice
constexpr int kSeqGroups = 2;   // 4 measured slower (more arrivals per hand-off)
constexpr int kSeqCols = 32 / kSeqGroups;
constexpr int kSeqThreads = 64 + 128 * kSeqGroups;

enum SeqBar : int {
    kA1Full = 0,   // [2] [Q~; W~] stage landed
    kA1Empty = 2,  // [2] R1 has read the stage
    kA2Full = 4,   // Mqk landed
    kA3Full = 5,   // K^ ^T landed
    kUtFull = 6,   // [2] U~ slice stage landed
    kUtEmpty = 8,  // [2] U~ slice read (one arrival per U warp)
    kR1Done = 10,
    kR2Done = 11,  // R2a complete: the state update may start, K^ ^T is free
    kODone = 12,   // R2b complete: output rows of D1 final, U^T and Mqk free
    kOFree = 13,   // the output warps have drained D1 of the previous chunk
    kUReady = 14,  // R2a issued (the producer then issues R2b)
    kFin = 15,     // completion of the MMA warp's MMAs
    kFinP = 16,    // completion of the producer's MMAs
    kSReady = 17,  // S^T published (one arrival per compute warp)
    kUPub = 18,    // U^T published (one arrival per U warp)
    kNumSeqBars = 19
};

template <int K, int V>
__global__ void __launch_bounds__(kSeqThreads, 1) chunk_seq_kernel(const uint8_t* __restrict__ recs, int64_t T, int Hv,
                                                           float scale, int NC, const float* state_in,
                                                           float* state_out, float* __restrict__ o,
                                                           unsigned int* __restrict__ o_amax,
                                                           unsigned int* __restrict__ err) {
    using L = SeqLayout<K>;
    using RC = ChunkRec<K, V>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024_shared(smem_raw);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar + kNumSeqBars);
    constexpr int NSL = V / 32;
    const int slice = blockIdx.x % NSL;
    const int h = (blockIdx.x / NSL) % Hv;
    const int b = blockIdx.x / (NSL * Hv);
    const int vs0 = slice * 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint8_t* rec0 = recs + (static_cast<int64_t>(b) * Hv + h) * NC * RC::BYTES;
    constexpr uint32_t IDESC = idesc_tf32(128, 32, false, false);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumSeqBars; ++i)
            mbar_init(&bar[i], i == kSReady                                                           ? 4 * kSeqGroups
                               : (i == kUtEmpty || i == kUtEmpty + 1 || i == kOFree || i == kUPub) ? 2 * kSeqGroups
                                                                                                     : 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    pdl_wait_and_trigger();

    if (warp == 0) {
        if (lane == 0) {
            // ---- producer: chunk records -> shared memory, and R2b (off the recurrence)
            auto load_a1 = [&](int c) {
                const int s = c & 1;
                mbar_arrive_expect_tx(&bar[kA1Full + s], L::A1_BYTES);
                for (uint32_t p = 0; p < L::A1_BYTES; p += 16384)
                    bulk_load(sm + L::A1 + s * L::A1_BYTES + p, rec0 + static_cast<int64_t>(c) * RC::BYTES + RC::A1 + p,
                              16384, &bar[kA1Full + s]);
            };
            auto load_ut = [&](int c) {
                const int s = c & 1;
                mbar_arrive_expect_tx(&bar[kUtFull + s], L::UT_BYTES);
                bulk_load(sm + L::UT + s * L::UT_BYTES,
                          rec0 + static_cast<int64_t>(c) * RC::BYTES + RC::UT + slice * RC::UT_SLICE, L::UT_BYTES,
                          &bar[kUtFull + s]);
            };
            auto load_m = [&](int c) {
                mbar_arrive_expect_tx(&bar[kA2Full], CH * CH * 4);
                bulk_load(sm + L::A23, rec0 + static_cast<int64_t>(c) * RC::BYTES + RC::A2, CH * CH * 4, &bar[kA2Full]);
            };
            auto load_kh = [&](int c) {
                mbar_arrive_expect_tx(&bar[kA3Full], RC::A3_BYTES);
                for (uint32_t p = 0; p < RC::A3_BYTES; p += 16384)
                    bulk_load(sm + L::A23 + CH * CH * 4 + p, rec0 + static_cast<int64_t>(c) * RC::BYTES + RC::A3 + p,
                              16384, &bar[kA3Full]);
            };
            // the sections of chunk c this CTA reads, pulled into L2 ahead of their copies
            auto prefetch = [&](int c) {
                const uint8_t* rc = rec0 + static_cast<int64_t>(c) * RC::BYTES;
                for (uint32_t p = 0; p < RC::UT; p += 16384) bulk_prefetch_l2(rc + p, 16384);
                bulk_prefetch_l2(rc + RC::UT + slice * RC::UT_SLICE, RC::UT_SLICE);
            };
            const uint32_t a2 = smem_u32(sm + L::A23), b2 = smem_u32(sm + L::B2);
            int last_a1 = 0, last_ut = 0, last_m = 0, last_kh = 0;   // last chunk issued to each buffer
            bool mma_issued = false;
            load_a1(0);
            load_ut(0);
            load_m(0);
            load_kh(0);
            if (NC > 1) {
                load_a1(1);
                load_ut(1);
                last_a1 = last_ut = 1;
            }
            for (int c = 1; c < 3 && c < NC; ++c) prefetch(c);
            for (int c = 0; c < NC; ++c) {
                const int s = c & 1;
                // R2b(c): D1[s] += Mqk U once U^T is published and R2a(c) has left the tensor
                // pipe (so R2b runs during the state update instead of ahead of it), with D1[s]
                // of chunk c-2 drained
                if (c + 3 < NC) prefetch(c + 3);
                bool w = mbar_wait(&bar[kUReady], c & 1, err, kErrTimeoutSeq) &&
                         mbar_wait(&bar[kR2Done], c & 1, err, kErrTimeoutSeq);
                if (!w) break;
                // R2a(c) has read K^ ^T: bring in the next chunk's
                if (c + 1 < NC) {
                    load_kh(c + 1);
                    last_kh = c + 1;
                }
                w = mbar_wait(&bar[kA2Full], c & 1, err, kErrTimeoutSeq) &&
                    (c == 0 || mbar_wait(&bar[kOFree], (c - 1) & 1, err, kErrTimeoutSeq));
                if (!w) break;
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < CH / 8; ++j)
                    mma_tf32_ss(tmem + 32 * s, sdesc_kmajor_sw128(a2 + (j >> 2) * CH * 128 + (j & 3) * 32),
                                sdesc_kmajor_sw128(b2 + (j >> 2) * 32 * 128 + (j & 3) * 32), IDESC, 1u);
                mma_commit(&bar[kODone]);
                mma_issued = true;
                // Mqk of chunk c+1 once R2b(c) has read this chunk's
                if (c + 1 < NC) {
                    if (!mbar_wait(&bar[kODone], c & 1, err, kErrTimeoutSeq)) break;
                    load_m(c + 1);
                    last_m = c + 1;
                }
                // [Q~; W~] and U~ of chunk c+2 into the stage chunk c used
                if (c + 2 < NC) {
                    if (!mbar_wait(&bar[kA1Empty + s], (c >> 1) & 1, err, kErrTimeoutSeq)) break;
                    load_a1(c + 2);
                    last_a1 = c + 2;
                    if (!mbar_wait(&bar[kUtEmpty + s], (c >> 1) & 1, err, kErrTimeoutSeq)) break;
                    load_ut(c + 2);
                    last_ut = c + 2;
                }
            }
            // every copy issued has landed, and every MMA issued here has completed, before exit
            // (stage s last received chunk last - (last - s) % 2, for the last chunk issued to it)
            for (int s = 0; s < 2; ++s) {
                const int ca = last_a1 - ((last_a1 - s) & 1), cu = last_ut - ((last_ut - s) & 1);
                if (ca >= 0) mbar_wait(&bar[kA1Full + s], (ca >> 1) & 1, err, kErrTimeoutSeq);
                if (cu >= 0) mbar_wait(&bar[kUtFull + s], (cu >> 1) & 1, err, kErrTimeoutSeq);
            }
            mbar_wait(&bar[kA2Full], last_m & 1, err, kErrTimeoutSeq);
            mbar_wait(&bar[kA3Full], last_kh & 1, err, kErrTimeoutSeq);
            if (mma_issued) {
                mma_commit(&bar[kFinP]);
                mbar_wait(&bar[kFinP], 0, err, kErrTimeoutSeq);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA warp: R1 and R2a, the two products on the recurrence
            const uint32_t b1 = smem_u32(sm + L::B1), b2 = smem_u32(sm + L::B2);
            const uint32_t a3 = smem_u32(sm + L::A23) + CH * CH * 4;
            for (int c = 0; c < NC; ++c) {
                const int s = c & 1;
                if (!mbar_wait(&bar[kSReady], c & 1, err, kErrTimeoutSeq) ||
                    !mbar_wait(&bar[kA1Full + s], (c >> 1) & 1, err, kErrTimeoutSeq))
                    break;
                tc_fence_after();
                const uint32_t a1 = smem_u32(sm + L::A1 + s * L::A1_BYTES);
#pragma unroll
                for (int j = 0; j < K / 8; ++j)
                    mma_tf32_ss(tmem + 32 * s, sdesc_kmajor_sw128(a1 + (j >> 2) * 128 * 128 + (j & 3) * 32),
                                sdesc_kmajor_sw128(b1 + (j >> 2) * 32 * 128 + (j & 3) * 32), IDESC, j > 0 ? 1u : 0u);
                mma_commit(&bar[kA1Empty + s]);
                mma_commit(&bar[kR1Done]);
                if (!mbar_wait(&bar[kUPub], c & 1, err, kErrTimeoutSeq) ||
                    !mbar_wait(&bar[kA3Full], c & 1, err, kErrTimeoutSeq))
                    break;
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < CH / 8; ++j)
                    mma_tf32_ss(tmem + 64, sdesc_kmajor_sw128(a3 + (j >> 2) * 128 * 128 + (j & 3) * 32),
                                sdesc_kmajor_sw128(b2 + (j >> 2) * 32 * 128 + (j & 3) * 32), IDESC, j > 0 ? 1u : 0u);
                mma_commit(&bar[kR2Done]);
                mbar_arrive(&bar[kUReady]);
            }
            // all MMAs issued here have completed before TMEM is released
            mma_commit(&bar[kFin]);
            mbar_wait(&bar[kFin], 0, err, kErrTimeoutSeq);
        }
    } else {
        // ---- compute warps: TMEM lane quarter q = warp % 4, columns c0..c0+kSeqCols-1 of the slice
        const int q = warp & 3;
        const int c0 = kSeqCols * ((warp - 2) >> 2);
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const int d = q * 32 + lane;             // state row
        const bool has_row = d < K;
        const bool u_role = q >= 2;              // W~ S0 of tokens 0..63 lands in lanes 64..127
        const int tu = d - 64;
        const int64_t sbase = (static_cast<int64_t>(b) * Hv + h) * K * V;
        // Byte offsets of (row c0 + i, column col) in a 32-row K-major swizzled image:
        // base + (i / 8) * 1024 + xo[i % 8] (only 8 swizzle patterns per column).
        auto swz_cols = [&](int col, uint32_t& base, uint32_t (&xo)[8]) {
            base = (col >> 5) * 32 * 128 + ((col & 3) << 2) + c0 * 128;
#pragma unroll
            for (int r = 0; r < 8; ++r) xo[r] = r * 128 + ((((col & 31) >> 2) ^ r) << 4);
        };
        uint8_t* b1p = sm + L::B1;
        uint8_t* b2p = sm + L::B2;
        uint32_t s_base = 0, s_xo[8];
        swz_cols(has_row ? d : 0, s_base, s_xo);
        uint32_t u_base = 0, u_xo[8];
        swz_cols(u_role ? tu : 0, u_base, u_xo);

        auto publish = [&](int bar_id) {
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[bar_id]);
        };
        // output rows t = d (lanes 0..63) of chunk c from D1
        auto drain_o = [&](int c, bool ok) -> bool {
            ok = __all_sync(0xffffffffu, ok && mbar_wait(&bar[kODone], c & 1, err, kErrTimeoutSeq));
            if (!ok) return false;
            tc_fence_after();
            uint32_t x[kSeqCols];
            tmem_ld_cols<kSeqCols>(tmem + 32 * (c & 1) + c0 + lane_base, x);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[kOFree]);
            const int64_t t = static_cast<int64_t>(c) * CH + d;
            float om = 0.0f;
            if (t < T) {
                float* orow = o + ((static_cast<int64_t>(b) * T + t) * Hv + h) * V + vs0 + c0;
#pragma unroll
                for (int v4 = 0; v4 < kSeqCols / 4; ++v4) {
                    const float4 ov = make_float4(scale * __uint_as_float(x[4 * v4]), scale * __uint_as_float(x[4 * v4 + 1]),
                                                  scale * __uint_as_float(x[4 * v4 + 2]),
                                                  scale * __uint_as_float(x[4 * v4 + 3]));
                    *reinterpret_cast<float4*>(orow + 4 * v4) = ov;
                    om = fmaxf(om, fmaxf(fmaxf(fabsf(ov.x), fabsf(ov.y)), fmaxf(fabsf(ov.z), fabsf(ov.w))));
                }
            }
            if (o_amax) {
                const unsigned int mb = __reduce_max_sync(0xffffffffu, __float_as_uint(om));
                if (lane == 0) atomicMax(o_amax, mb);
            }
            return true;
        };

        float S[kSeqCols];
#pragma unroll
        for (int v4 = 0; v4 < kSeqCols / 4; ++v4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (state_in && has_row)
                x = *reinterpret_cast<const float4*>(state_in + sbase + static_cast<int64_t>(d) * V + vs0 + c0 + 4 * v4);
            S[4 * v4] = x.x; S[4 * v4 + 1] = x.y; S[4 * v4 + 2] = x.z; S[4 * v4 + 3] = x.w;
        }
        if (has_row) {
#pragma unroll
            for (int i = 0; i < kSeqCols; ++i)
                *reinterpret_cast<float*>(b1p + s_base + (i >> 3) * 1024 + s_xo[i & 7]) = __uint_as_float(to_tf32(S[i]));
        }
        publish(kSReady);
        bool ok = true;
        for (int c = 0; c < NC && ok; ++c) {
            const int s = c & 1;
            const float gc = *reinterpret_cast<const float*>(rec0 + static_cast<int64_t>(c) * RC::BYTES + RC::GC);
            if (u_role) {
                float ut[kSeqCols];
                ok = __all_sync(0xffffffffu, mbar_wait(&bar[kUtFull + s], (c >> 1) & 1, err, kErrTimeoutSeq));
                if (!ok) break;
                const uint8_t* up = sm + L::UT + s * L::UT_BYTES + tu * 128;
#pragma unroll
                for (int jj = 0; jj < kSeqCols / 4; ++jj) {
                    const int j = (c0 >> 2) + jj;
                    const float4 x = *reinterpret_cast<const float4*>(up + ((j ^ (tu & 7)) << 4));
                    ut[4 * jj] = x.x; ut[4 * jj + 1] = x.y; ut[4 * jj + 2] = x.z; ut[4 * jj + 3] = x.w;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[kUtEmpty + s]);
                // R1 done; R2b of the previous chunk has finished reading U^T
                ok = __all_sync(0xffffffffu, mbar_wait(&bar[kR1Done], c & 1, err, kErrTimeoutSeq) &&
                                                 (c == 0 || mbar_wait(&bar[kODone], (c - 1) & 1, err, kErrTimeoutSeq)));
                if (!ok) break;
                tc_fence_after();
                uint32_t x[kSeqCols];
                tmem_ld_cols<kSeqCols>(tmem + 32 * s + c0 + lane_base, x);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < kSeqCols; ++i)
                    *reinterpret_cast<float*>(b2p + u_base + (i >> 3) * 1024 + u_xo[i & 7]) =
                        __uint_as_float(to_tf32(ut[i] - __uint_as_float(x[i])));
                publish(kUPub);
            } else if (c > 0) {
                ok = drain_o(c - 1, ok);
                if (!ok) break;
            }
            ok = __all_sync(0xffffffffu, mbar_wait(&bar[kR2Done], c & 1, err, kErrTimeoutSeq));
            if (!ok) break;
            tc_fence_after();
            uint32_t x[kSeqCols];
            tmem_ld_cols<kSeqCols>(tmem + 64 + c0 + lane_base, x);
            tmem_wait_ld();
            if (has_row) {
                const float eg = expf(gc);
#pragma unroll
                for (int i = 0; i < kSeqCols; ++i) {
                    S[i] = fmaf(eg, S[i], __uint_as_float(x[i]));
                    *reinterpret_cast<float*>(b1p + s_base + (i >> 3) * 1024 + s_xo[i & 7]) =
                        __uint_as_float(to_tf32(S[i]));
                }
            }
            publish(kSReady);
        }
        if (ok && !u_role) ok = drain_o(NC - 1, ok);
        if (ok && state_out && has_row) {
#pragma unroll
            for (int v4 = 0; v4 < kSeqCols / 4; ++v4)
                *reinterpret_cast<float4*>(state_out + sbase + static_cast<int64_t>(d) * V + vs0 + c0 + 4 * v4) =
                    make_float4(S[4 * v4], S[4 * v4 + 1], S[4 * v4 + 2], S[4 * v4 + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

template <int K, int V>
nvfp4_status launch_chunked_kv(const float* q, const float* k, const float* v, int64_t ld_v, const float* g,
                               const float* beta, int B, int64_t T, const gdn_dims& d, float scale, int form,
                               const float* s_in, float* s_out, float* o, void* ws, unsigned int* o_amax,
                               int64_t ld_qk, int normalize_qk, cudaStream_t st) {
    const int NC = static_cast<int>((T + CH - 1) / CH);
    const int prep_smem = sizeof(PrepSmem<K, V>);
    const int seq_smem = SeqLayout<K>::BYTES;
    static PerDeviceOnce attr_once;
    nvfp4_status s = once_per_device(attr_once, [&]() -> nvfp4_status {
        cudaError_t e = cudaFuncSetAttribute(chunk_prep_kernel<K, V>, cudaFuncAttributeMaxDynamicSharedMemorySize, prep_smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prep)");
        e = cudaFuncSetAttribute(chunk_seq_kernel<K, V>, cudaFuncAttributeMaxDynamicSharedMemorySize, seq_smem);
        return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "cudaFuncSetAttribute(seq)");
    });
    if (s != NVFP4_OK) return s;
    unsigned int* err = device_error_word();
    if (!err) return fail(NVFP4_ERR_CUDA, "device error word unavailable");
    uint8_t* recs = static_cast<uint8_t*>(ws);
    const unsigned prep_blocks = static_cast<unsigned>(static_cast<int64_t>(B) * NC * d.Hv);
    cudaError_t e = launch_pdl(chunk_prep_kernel<K, V>, dim3(prep_blocks), dim3(256), prep_smem, st, q, k, ld_qk,
                               normalize_qk, v, ld_v, g, beta, T, d.Hk, d.Hv, form, NC, recs);
    if (e != cudaSuccess) return cuda_fail(e, "chunked scan launch");
    const unsigned seq_blocks = static_cast<unsigned>(B * d.Hv * (V / 32));
    e = launch_pdl(chunk_seq_kernel<K, V>, dim3(seq_blocks), dim3(kSeqThreads), seq_smem, st, recs, T, d.Hv, scale, NC,
                   s_in, s_out, o, o_amax, err);
    if (e != cudaSuccess) return cuda_fail(e, "chunked scan launch");
    return NVFP4_OK;
}

// Zero the U~ sections of n_rec records: only U~ = T diag(beta) V depends on v,
// so the records become those of the same span with v = 0.
template <int K, int V>
__global__ void __launch_bounds__(256) zero_ut_kernel(uint8_t* __restrict__ recs, int64_t n_rec) {
    pdl_wait_and_trigger();
    using RC = ChunkRec<K, V>;
    constexpr int64_t per = static_cast<int64_t>(V / 32) * RC::UT_SLICE / 16;   // 16-byte words per record
    const int64_t total = n_rec * per;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = e / per, i = e - r * per;
        reinterpret_cast<float4*>(recs + r * RC::BYTES + RC::UT)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// One span's zero-start scan (o, S_loc) and its maps (P, qmap) with one chunk
// preparation: the sequential kernel runs on the records as prepared, then on
// the same records with U~ zeroed, from P = I (K == V only).
template <int K>
nvfp4_status launch_span_chunked(const float* q, const float* k, const float* v, int64_t ld_v, const float* g,
                                 const float* beta, int B, int64_t T, const gdn_dims& d, float scale, int form,
                                 float* o, float* S_loc, float* P, float* qmap, void* ws, cudaStream_t st) {
    nvfp4_status s = launch_chunked_kv<K, K>(q, k, v, ld_v, g, beta, B, T, d, scale, form, nullptr, S_loc, o, ws,
                                             nullptr, static_cast<int64_t>(d.Hk) * K, 0, st);
    if (s != NVFP4_OK) return s;
    const int NC = static_cast<int>((T + CH - 1) / CH);
    const int64_t n_rec = static_cast<int64_t>(B) * d.Hv * NC;
    uint8_t* recs = static_cast<uint8_t*>(ws);
    const int64_t words = n_rec * (K / 32) * ChunkRec<K, K>::UT_SLICE / 16;
    const unsigned zb = static_cast<unsigned>(std::min<int64_t>((words + 255) / 256, int64_t(num_sms()) * 8));
    cudaError_t e = launch_pdl(zero_ut_kernel<K, K>, dim3(zb), dim3(256), 0, st, recs, n_rec);
    if (e != cudaSuccess) return cuda_fail(e, "record U~ zero launch");
    if ((s = identity_fill_launch(P, static_cast<int64_t>(B) * d.Hv, K, nullptr, 0, st)) != NVFP4_OK) return s;
    unsigned int* err = device_error_word();
    if (!err) return fail(NVFP4_ERR_CUDA, "device error word unavailable");
    e = launch_pdl(chunk_seq_kernel<K, K>, dim3(static_cast<unsigned>(B * d.Hv * (K / 32))), dim3(kSeqThreads),
                   static_cast<int>(SeqLayout<K>::BYTES), st, recs, T, d.Hv, scale, NC, P, P, qmap,
                   static_cast<unsigned int*>(nullptr), err);
    if (e != cudaSuccess) return cuda_fail(e, "chunked scan launch");
    return NVFP4_OK;
}

size_t chunk_rec_bytes(const gdn_dims& d) {
    if (d.K == 128 && d.V == 128) return ChunkRec<128, 128>::BYTES;
    if (d.K == 128 && d.V == 64) return ChunkRec<128, 64>::BYTES;
    if (d.K == 64 && d.V == 128) return ChunkRec<64, 128>::BYTES;
    return ChunkRec<64, 64>::BYTES;
}

}  // namespace

nvfp4_status validate_dims(const gdn_dims* d);

size_t scan_workspace_bytes(int B, int64_t T, const gdn_dims& d, int algo) {
    const bool chunked = algo == GDN_SCAN_CHUNKED || (algo == GDN_SCAN_AUTO && T > 1);
    if (!chunked) return 0;
    const int64_t NC = (T + CH - 1) / CH;
    return static_cast<size_t>(B) * d.Hv * NC * chunk_rec_bytes(d);
}

nvfp4_status scan_launch(const float* q, const float* k, const float* v, int64_t ld_v, const float* g,
                         const float* beta, int B, int64_t T, const gdn_dims& d, float scale, int form, int algo,
                         const float* s_in, float* s_out, float* o, void* ws, cudaStream_t st,
                         unsigned int* o_amax, int64_t ld_qk, int normalize_qk) {
    const bool chunked = algo == GDN_SCAN_CHUNKED || (algo == GDN_SCAN_AUTO && T > 1);
    if (!chunked) {
        const unsigned blocks = static_cast<unsigned>(B * d.Hv * (d.V / 32));
        const cudaError_t e =
            d.K == 128 ? launch_pdl(scan_recurrent_kernel<128>, dim3(blocks), dim3(128), 0, st, q, k, ld_qk,
                                    normalize_qk, v, ld_v, g, beta, B, T, d.Hk, d.Hv, d.V, scale, form, s_in, s_out, o,
                                    o_amax)
                       : launch_pdl(scan_recurrent_kernel<64>, dim3(blocks), dim3(128), 0, st, q, k, ld_qk,
                                    normalize_qk, v, ld_v, g, beta, B, T, d.Hk, d.Hv, d.V, scale, form, s_in, s_out, o,
                                    o_amax);
        if (e != cudaSuccess) return cuda_fail(e, "recurrent scan launch");
        return NVFP4_OK;
    }
    if (d.K == 128 && d.V == 128)
        return launch_chunked_kv<128, 128>(q, k, v, ld_v, g, beta, B, T, d, scale, form, s_in, s_out, o, ws, o_amax, ld_qk, normalize_qk, st);
    if (d.K == 128 && d.V == 64)
        return launch_chunked_kv<128, 64>(q, k, v, ld_v, g, beta, B, T, d, scale, form, s_in, s_out, o, ws, o_amax, ld_qk, normalize_qk, st);
    if (d.K == 64 && d.V == 128)
        return launch_chunked_kv<64, 128>(q, k, v, ld_v, g, beta, B, T, d, scale, form, s_in, s_out, o, ws, o_amax, ld_qk, normalize_qk, st);
    return launch_chunked_kv<64, 64>(q, k, v, ld_v, g, beta, B, T, d, scale, form, s_in, s_out, o, ws, o_amax, ld_qk, normalize_qk, st);
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
    if (!aligned16(state_in) || !aligned16(state_out))   // the chunked kernel moves the state as float4
        return fail(NVFP4_ERR_MISALIGNED, "state_in and state_out must be 16-byte aligned");
    const size_t need = scan_workspace_bytes(B, T, *dims, algo);
    if (need && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255)))
        return fail(NVFP4_ERR_WORKSPACE, "scan workspace missing, too small or not 256-byte aligned");
    return scan_launch(q_hat, k_hat, v, ld_v, g, beta, B, T, *dims, scale, form, algo, state_in, state_out, o,
                       workspace, as_stream(stream), nullptr, static_cast<int64_t>(dims->Hk) * dims->K, 0);
}

extern "C" size_t gdn_scan_span_workspace_size(int32_t B, int64_t T, const gdn_dims* dims, int32_t algo) {
    if (!dims || nvg::validate_dims(dims) != NVFP4_OK || B < 1 || T < 1) return 0;
    return std::max(nvg::scan_workspace_bytes(B, T, *dims, algo), nvg::transition_workspace_bytes(B, T, *dims, algo));
}

extern "C" nvfp4_status gdn_scan_span(const float* q_hat, const float* k_hat, const float* v, int64_t ld_v,
                                      const float* g, const float* beta, int32_t B, int64_t T, const gdn_dims* dims,
                                      float scale, int32_t form, int32_t algo, float* o, float* S_loc, float* P,
                                      float* qmap, void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
    using namespace nvg;
    nvfp4_status s = validate_dims(dims);
    if (s != NVFP4_OK) return s;
    if (!q_hat || !k_hat || !v || !g || !beta || !o || !S_loc || !P || !qmap)
        return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
    if (B < 1 || T < 1) return fail(NVFP4_ERR_INVALID_ARG, "B and T must be >= 1");
    if (form != GDN_FORM_PAGES && form != GDN_FORM_STANDARD) return fail(NVFP4_ERR_INVALID_ARG, "bad form");
    if (algo != GDN_SCAN_AUTO && algo != GDN_SCAN_RECURRENT && algo != GDN_SCAN_CHUNKED)
        return fail(NVFP4_ERR_INVALID_ARG, "bad algo");
    if (ld_v < static_cast<int64_t>(dims->Hv) * dims->V) return fail(NVFP4_ERR_INVALID_ARG, "ld_v < Hv*V");
    if (static_cast<int64_t>(B) * T > (int64_t(1) << 31)) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "B*T too large");
    if (!aligned16(q_hat) || !aligned16(k_hat) || !aligned16(v) || ld_v % 4 || !aligned16(o) || !aligned16(S_loc) ||
        !aligned16(P) || !aligned16(qmap))
        return fail(NVFP4_ERR_MISALIGNED, "pointers must be 16-byte aligned and ld_v % 4 == 0");
    const size_t need = std::max(scan_workspace_bytes(B, T, *dims, algo), transition_workspace_bytes(B, T, *dims, algo));
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return fail(NVFP4_ERR_WORKSPACE, "span workspace missing, too small or not 256-byte aligned");
    const size_t nbytes[5] = {static_cast<size_t>(B) * T * dims->Hv * dims->V * 4,
                              static_cast<size_t>(B) * dims->Hv * dims->K * dims->V * 4,
                              static_cast<size_t>(B) * dims->Hv * dims->K * dims->K * 4,
                              static_cast<size_t>(B) * T * dims->Hv * dims->K * 4, need};
    const char* ptrs[5] = {reinterpret_cast<const char*>(o), reinterpret_cast<const char*>(S_loc),
                           reinterpret_cast<const char*>(P), reinterpret_cast<const char*>(qmap),
                           static_cast<const char*>(workspace)};
    for (int i = 0; i < 5; ++i)
        for (int j = i + 1; j < 5; ++j)
            if (ptrs[i] < ptrs[j] + nbytes[j] && ptrs[j] < ptrs[i] + nbytes[i])
                return fail(NVFP4_ERR_INVALID_ARG, "o, S_loc, P, qmap and the workspace must not overlap");
    const cudaStream_t st = as_stream(stream);
    const bool chunked = algo == GDN_SCAN_CHUNKED || (algo == GDN_SCAN_AUTO && T > 1);
    const int64_t ld_qk = static_cast<int64_t>(dims->Hk) * dims->K;
    if (chunked && dims->K == dims->V) {
        if (dims->K == 128)
            return launch_span_chunked<128>(q_hat, k_hat, v, ld_v, g, beta, B, T, *dims, scale, form, o, S_loc, P,
                                            qmap, workspace, st);
        return launch_span_chunked<64>(q_hat, k_hat, v, ld_v, g, beta, B, T, *dims, scale, form, o, S_loc, P, qmap,
                                       workspace, st);
    }
    // the zero-start scan, then the maps (the scan on v = 0 from P = I with V = K) in the same workspace
    if ((s = scan_launch(q_hat, k_hat, v, ld_v, g, beta, B, T, *dims, scale, form, algo, nullptr, S_loc, o,
                         workspace, st, nullptr, ld_qk, 0)) != NVFP4_OK)
        return s;
    gdn_dims dk = *dims;
    dk.V = dims->K;
    const size_t zero_off = (scan_workspace_bytes(B, T, dk, algo) + 255) / 256 * 256;
    float* zero_row = reinterpret_cast<float*>(static_cast<char*>(workspace) + zero_off);
    if ((s = identity_fill_launch(P, static_cast<int64_t>(B) * dims->Hv, dims->K, zero_row,
                                  static_cast<int64_t>(dims->Hv) * dims->K, st)) != NVFP4_OK)
        return s;
    return scan_launch(q_hat, k_hat, zero_row, 0, g, beta, B, T, dk, scale, form, algo, P, P, qmap, workspace, st,
                       nullptr, ld_qk, 0);
}
