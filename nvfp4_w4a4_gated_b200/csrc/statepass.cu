// statepass.cu -- joining spans of one sequence through the recurrence's state.
//
// The delta-rule update of Eq.(2) (review page "Why Gated DeltaNet Survives
// 4-Bit Quantization", background) is affine in the state: one token maps S to
// A_t S + b_t k_t v_t^T with A_t = a_t I - b_t k_t k_t^T (the pages' form) or
// a_t (I - b_t k_t k_t^T) (decay inside).  A span of tokens therefore maps an
// initial state S_in to P S_in + S_loc, where P = A_T ... A_1 and S_loc is the
// span's final state from a zero start, and each output of the span gains
// S_in^T m_t with m_t = scale P_t^T q_t.  A sequence split into spans (one per
// GPU, say) is scanned span by span from zero in parallel; the spans' maps are
// then composed in order to give each span its true initial state, and the
// outputs are corrected.
//
//   gdn_scan_transition   P and m of a span: the chunked (or one-token) scan
//                         run on v = 0 from S_in = I with V = K, so P is its
//                         final state and m its output;
//   gdn_state_combine     S_out = P S_in + S_loc per (sequence, value head),
//                         or a chain of m such steps in one launch;
//   gdn_scan_correct      o_t += S_in^T m_t over a span's tokens, with the
//                         quantiser's amax of the corrected o folded in.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "common.cuh"

namespace nvg {

nvfp4_status validate_dims(const gdn_dims* d);
size_t scan_workspace_bytes(int B, int64_t T, const gdn_dims& d, int algo);
nvfp4_status scan_launch(const float* q, const float* k, const float* v, int64_t ld_v, const float* g,
                         const float* beta, int B, int64_t T, const gdn_dims& d, float scale, int form, int algo,
                         const float* s_in, float* s_out, float* o, void* ws, cudaStream_t st,
                         unsigned int* o_amax, int64_t ld_qk, int normalize_qk);

namespace {

constexpr size_t kAlign = 256;
inline size_t round_up(size_t n) { return (n + kAlign - 1) / kAlign * kAlign; }

// P[n] = I (K x K) for every (sequence, value head) and a zero row of Hv*K floats.
__global__ void __launch_bounds__(256) identity_fill_kernel(float* __restrict__ P, int64_t n_mat, int K,
                                                            float* __restrict__ zero_row, int64_t n_zero) {
    pdl_wait_and_trigger();
    const int64_t total = n_mat * K * K;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += stride) {
        const int64_t rc = e % (static_cast<int64_t>(K) * K);
        P[e] = (rc / K == rc % K) ? 1.0f : 0.0f;
    }
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n_zero; e += stride)
        zero_row[e] = 0.0f;
}

// The chain S = S_in; S = P[j] S + S_loc[j] for j = 0..m-1; S_out = S, per
// (sequence, value head) n.  The columns of S evolve independently, so one CTA
// per (n, 32 columns) carries its K x 32 slice through the whole chain in
// shared memory.  P[j+1][n] (K x K) is copied asynchronously into the second of
// two shared buffers while step j computes; rows are padded by 4 floats so the
// four consecutive rows a warp reads at once fall in different banks.  Thread
// (tr, tc) of 256 owns rows tr + 32 r (r < K / 32) and columns 4 tc .. 4 tc + 3.
constexpr int kChainCols = 32;
template <int K>
__global__ void __launch_bounds__(256, 1) state_chain_kernel(const float* __restrict__ P, const float* S_loc,
                                                             const float* S_in, float* S_out, int m,
                                                             int64_t n_total, int V) {
    pdl_wait_and_trigger();
    constexpr int NT = 256;            // threads
    constexpr int R = K / 32;          // rows per thread
    constexpr int RS = 32;             // row stride between a thread's rows
    constexpr int PK = K + 4;
    extern __shared__ __align__(16) float smem[];
    float* Pb = smem;                      // [2][K][K + 4]
    float* Ss = smem + 2 * K * PK;         // [K][32]
    const int64_t n = blockIdx.x;
    const int c0 = blockIdx.y * kChainCols;
    const int tc = threadIdx.x & 7, tr = threadIdx.x >> 3;
    auto issue_p = [&](int j, int buf) {
        const float* Pj = P + (static_cast<int64_t>(j) * n_total + n) * K * K;
        float* dst = Pb + buf * K * PK;
#pragma unroll 4
        for (int e = threadIdx.x; e < K * K / 4; e += NT) {
            const int i = e / (K / 4), l4 = e - i * (K / 4);
            cp_async16(dst + i * PK + 4 * l4, Pj + 4 * static_cast<int64_t>(e), true);
        }
        cp_async_commit();
    };
    issue_p(0, 0);
    for (int e = threadIdx.x; e < K * kChainCols; e += NT) {
        const int i = e >> 5, cc = e & 31;
        Ss[e] = S_in ? S_in[(n * K + i) * V + c0 + cc] : 0.0f;
    }
    for (int j = 0; j < m; ++j) {
        if (j + 1 < m) issue_p(j + 1, (j + 1) & 1);
        else cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();   // P[j] landed everywhere; the slice of the previous step is written
        const float* Ps = Pb + (j & 1) * K * PK;
        float acc[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) acc[r][cc] = 0.0f;
#pragma unroll 2
        for (int l = 0; l < K; l += 4) {
            float4 p[R];
#pragma unroll
            for (int r = 0; r < R; ++r) p[r] = *reinterpret_cast<const float4*>(Ps + (tr + RS * r) * PK + l);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 sv = *reinterpret_cast<const float4*>(Ss + (l + q) * kChainCols + 4 * tc);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float pv = q == 0 ? p[r].x : q == 1 ? p[r].y : q == 2 ? p[r].z : p[r].w;
                    acc[r][0] = fmaf(pv, sv.x, acc[r][0]);
                    acc[r][1] = fmaf(pv, sv.y, acc[r][1]);
                    acc[r][2] = fmaf(pv, sv.z, acc[r][2]);
                    acc[r][3] = fmaf(pv, sv.w, acc[r][3]);
                }
            }
        }
        __syncthreads();   // every thread has read the old slice and P[j]
        const float* Lj = S_loc ? S_loc + (static_cast<int64_t>(j) * n_total + n) * K * V : nullptr;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int i = tr + RS * r;
            float4 add = make_float4(0.f, 0.f, 0.f, 0.f);
            if (Lj) {
                const float* lp = Lj + static_cast<int64_t>(i) * V + c0 + 4 * tc;
                add = make_float4(lp[0], lp[1], lp[2], lp[3]);
            }
            *reinterpret_cast<float4*>(Ss + i * kChainCols + 4 * tc) =
                make_float4(acc[r][0] + add.x, acc[r][1] + add.y, acc[r][2] + add.z, acc[r][3] + add.w);
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    for (int e = threadIdx.x; e < K * kChainCols; e += NT) {
        const int i = e >> 5, cc = e & 31;
        S_out[(n * K + i) * V + c0 + cc] = Ss[e];
    }
}

template <int K>
nvfp4_status launch_chain(const float* P, const float* S_loc, const float* S_in, float* S_out, int m, int64_t n,
                          int V, cudaStream_t st) {
    constexpr int smem = (2 * K * (K + 4) + K * kChainCols) * 4;
    static PerDeviceOnce attr_once;
    const nvfp4_status s = smem_limit_once(attr_once, state_chain_kernel<K>, smem, "cudaFuncSetAttribute(chain)");
    if (s != NVFP4_OK) return s;
    const cudaError_t e = launch_pdl(state_chain_kernel<K>, dim3(static_cast<unsigned>(n), V / kChainCols),
                                     dim3(256), smem, st, P, S_loc, S_in, S_out, m, n, V);
    if (e != cudaSuccess) return cuda_fail(e, "state combine launch");
    return NVFP4_OK;
}

// o[b,t,h,:] += S_in[b,h]^T m[b,t,h,:].  The work is a list of items (b, h,
// tile of 32 tokens) in that order; each CTA takes a contiguous run of items,
// so it stages S_in[b,h] (K x V) in shared memory once per head it meets.  The
// m rows of the next item are copied asynchronously (double buffer) while the
// current item computes, and each thread loads its o values before the k loop.
// Thread (ty, tx) of a 16 x 16 grid owns tokens 2ty, 2ty+1 and the columns
// 4tx + 64c .. +3 (c < V/64).  The largest |o| of the CTA goes into the
// quantiser's amax word with one atomicMax.
constexpr int kCorrTok = 32;
template <int K, int V>
__global__ void __launch_bounds__(256, 2) scan_correct_kernel(const float* __restrict__ m,
                                                              const float* __restrict__ S_in, float* __restrict__ o,
                                                              int64_t T, int Hv, int64_t n_items, int per_cta,
                                                              unsigned int* __restrict__ o_amax) {
    pdl_wait_and_trigger();
    constexpr int VC = V / 64;
    extern __shared__ __align__(16) float smem[];
    float* Ss = smem;              // [K][V]
    float* Mb = smem + K * V;      // [2][kCorrTok][K]
    const int64_t tiles = (T + kCorrTok - 1) / kCorrTok;
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * per_cta;
    const int64_t i1 = i0 + per_cta < n_items ? i0 + per_cta : n_items;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float mx = 0.0f;
    if (i0 < i1) {
        auto stage_S = [&](int64_t bh) {
            const float4* S4 = reinterpret_cast<const float4*>(S_in + bh * K * V);
            for (int e = threadIdx.x; e < K * V / 4; e += 256) reinterpret_cast<float4*>(Ss)[e] = S4[e];
        };
        auto issue_m = [&](int64_t item, int buf) {
            const int64_t bh = item / tiles, t0 = (item - bh * tiles) * kCorrTok;
            const int64_t b = bh / Hv, h = bh - b * Hv;
            float* dst = Mb + buf * kCorrTok * K;
            for (int e = threadIdx.x; e < kCorrTok * K / 4; e += 256) {
                const int r = e / (K / 4), c4 = e - r * (K / 4);
                const int64_t t = t0 + r;
                const bool valid = t < T;
                cp_async16(dst + 4 * e, valid ? m + ((b * T + t) * Hv + h) * K + 4 * c4 : m, valid);
            }
            cp_async_commit();
        };
        int64_t cur_bh = i0 / tiles;
        stage_S(cur_bh);
        issue_m(i0, 0);
        for (int64_t it = i0; it < i1; ++it) {
            const int buf = static_cast<int>((it - i0) & 1);
            if (it + 1 < i1) issue_m(it + 1, buf ^ 1);
            else cp_async_commit();                    // one group per iteration
            cp_async_wait<1>();                          // this item's rows have landed
            __syncthreads();
            const int64_t bh = it / tiles, t0 = (it - bh * tiles) * kCorrTok;
            const int64_t b = bh / Hv, h = bh - b * Hv;
            float4 ov[2][VC];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int64_t t = t0 + 2 * ty + r;
#pragma unroll
                for (int c = 0; c < VC; ++c)
                    ov[r][c] = t < T ? *reinterpret_cast<const float4*>(o + ((b * T + t) * Hv + h) * V + 4 * tx + 64 * c)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            const float* Ms = Mb + buf * kCorrTok * K;
            float acc[2][4 * VC];
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int c = 0; c < 4 * VC; ++c) acc[r][c] = 0.0f;
#pragma unroll 4
            for (int kk = 0; kk < K; kk += 4) {
                const float4 a0 = *reinterpret_cast<const float4*>(Ms + (2 * ty) * K + kk);
                const float4 a1 = *reinterpret_cast<const float4*>(Ms + (2 * ty + 1) * K + kk);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float x0 = q == 0 ? a0.x : q == 1 ? a0.y : q == 2 ? a0.z : a0.w;
                    const float x1 = q == 0 ? a1.x : q == 1 ? a1.y : q == 2 ? a1.z : a1.w;
#pragma unroll
                    for (int c = 0; c < VC; ++c) {
                        const float4 sv = *reinterpret_cast<const float4*>(Ss + (kk + q) * V + 4 * tx + 64 * c);
                        acc[0][4 * c + 0] = fmaf(x0, sv.x, acc[0][4 * c + 0]);
                        acc[0][4 * c + 1] = fmaf(x0, sv.y, acc[0][4 * c + 1]);
                        acc[0][4 * c + 2] = fmaf(x0, sv.z, acc[0][4 * c + 2]);
                        acc[0][4 * c + 3] = fmaf(x0, sv.w, acc[0][4 * c + 3]);
                        acc[1][4 * c + 0] = fmaf(x1, sv.x, acc[1][4 * c + 0]);
                        acc[1][4 * c + 1] = fmaf(x1, sv.y, acc[1][4 * c + 1]);
                        acc[1][4 * c + 2] = fmaf(x1, sv.z, acc[1][4 * c + 2]);
                        acc[1][4 * c + 3] = fmaf(x1, sv.w, acc[1][4 * c + 3]);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int64_t t = t0 + 2 * ty + r;
                if (t < T) {
#pragma unroll
                    for (int c = 0; c < VC; ++c) {
                        float4 x = ov[r][c];
                        x.x += acc[r][4 * c + 0];
                        x.y += acc[r][4 * c + 1];
                        x.z += acc[r][4 * c + 2];
                        x.w += acc[r][4 * c + 3];
                        *reinterpret_cast<float4*>(o + ((b * T + t) * Hv + h) * V + 4 * tx + 64 * c) = x;
                        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
                    }
                }
            }
            __syncthreads();                             // this item's rows and S are no longer read
            if (it + 1 < i1 && (it + 1) / tiles != cur_bh) {
                cur_bh = (it + 1) / tiles;
                stage_S(cur_bh);                         // visible after the next iteration's barrier
            }
        }
        cp_async_wait<0>();
    }
    if (o_amax) {
        __shared__ unsigned int wmax[8];
        const unsigned int wm = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
        if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = wm;
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned int bm = wmax[0];
#pragma unroll
            for (int i = 1; i < 8; ++i) bm = bm > wmax[i] ? bm : wmax[i];
            atomicMax(o_amax, bm);
        }
    }
}

template <int K, int V>
nvfp4_status launch_correct(const float* m, const float* S_in, float* o, int B, int64_t T, int Hv,
                            unsigned int* o_amax, cudaStream_t st) {
    constexpr int smem = (K * V + 2 * kCorrTok * K) * 4;
    static PerDeviceOnce attr_once;
    const nvfp4_status s = smem_limit_once(attr_once, scan_correct_kernel<K, V>, smem, "cudaFuncSetAttribute(correct)");
    if (s != NVFP4_OK) return s;
    const int64_t n_items = static_cast<int64_t>(B) * Hv * ((T + kCorrTok - 1) / kCorrTok);
    const int64_t slots = int64_t(num_sms()) * 2;
    const int per_cta = static_cast<int>((n_items + slots - 1) / slots);
    const unsigned grid = static_cast<unsigned>((n_items + per_cta - 1) / per_cta);
    const cudaError_t e = launch_pdl(scan_correct_kernel<K, V>, dim3(grid), dim3(256), smem, st, m, S_in, o, T, Hv,
                                     n_items, per_cta, o_amax);
    if (e != cudaSuccess) return cuda_fail(e, "scan correct launch");
    return NVFP4_OK;
}

// The same correction on the tcgen05 tensor cores (kind::tf32, float32
// accumulation in TMEM): per item (b, h, tile of 128 tokens)
//   D[t, j] = sum_i m[t, i] S_in[i, j]     (M = 128 tokens, N = V, K)
// with A = the tile's m rows and B = S_in^T (the V columns as rows), both in
// 128-byte-swizzled K-major images and rounded to TF32 (nearest).  One CTA per
// SM takes a contiguous run of items (tile fastest) and stages S_in^T once per
// head; the m rows of the next item are copied asynchronously into the other A
// buffer while the current item's MMAs and epilogue run.  The accumulator drains
// through the current A buffer (warp w of 16 reads TMEM lanes 32 (w % 4) .. + 31,
// one token each, and columns V/4 (w / 4) .. + V/4 - 1, and writes them as
// row-swizzled 16-byte chunks), so o is read and written in whole rows; the o
// loads are issued while the MMAs run.  The MMA completion wait is
// bounded; on expiry the CTA records kErrTimeoutCorrect and stops.
__device__ __forceinline__ uint32_t sw128_off(int r, int col, int rows) {
    return static_cast<uint32_t>((col >> 5) * rows * 128 + r * 128 + ((((col & 31) >> 2) ^ (r & 7)) << 4) +
                                 ((col & 3) << 2));
}
__device__ __forceinline__ float tf32_rn(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

constexpr int kTcTok = 128;     // tokens per item (MMA M)

template <int K, int V>
struct CorrTcLayout {
    static constexpr uint32_t A_BYTES = kTcTok * (K > V ? K : V) * 4;
    static constexpr uint32_t A = 0;     // two [128 tokens x K] images; the drained D tile reuses one
    static constexpr uint32_t Bm = A + 2 * A_BYTES;            // [V columns x K] image
    static constexpr uint32_t B_BYTES = V * K * 4;
    static constexpr uint32_t BAR = Bm + B_BYTES;
    static constexpr uint32_t BYTES = BAR + 64 + 1024;         // + alignment slack
};

template <int K, int V>
__global__ void __launch_bounds__(512, 1) scan_correct_tc_kernel(const float* __restrict__ m,
                                                                 const float* __restrict__ S_in,
                                                                 float* __restrict__ o, int64_t T, int Hv,
                                                                 int64_t n_items, int per_cta,
                                                                 unsigned int* __restrict__ o_amax,
                                                                 unsigned int* __restrict__ err) {
    using L = CorrTcLayout<K, V>;
    constexpr uint32_t IDESC = idesc_tf32(kTcTok, V, false, false);
    constexpr int NT = 512;
    constexpr int CPT = kTcTok * K / 4 / NT;        // 16-byte chunks of A per thread
    constexpr int COLS = V / 4;                     // columns per warp
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024_shared(smem_raw);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + L::BAR + 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_holder, V);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    pdl_wait_and_trigger();

    const int64_t tiles = (T + kTcTok - 1) / kTcTok;
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * per_cta;
    const int64_t i1 = i0 + per_cta < n_items ? i0 + per_cta : n_items;
    const int q = warp & 3, cg = warp >> 2;
    // this thread's A chunks: e = u * NT + tid -> row e / (K/4), column 4 (e % (K/4))
    auto issue_a = [&](int64_t item, int buf) {
        const int64_t bh = item / tiles, t0 = (item - bh * tiles) * kTcTok;
        const int64_t b = bh / Hv, h = bh - b * Hv;
        uint8_t* dst = sm + L::A + buf * L::A_BYTES;
#pragma unroll
        for (int u = 0; u < CPT; ++u) {
            const int e = u * NT + threadIdx.x;
            const int r = e / (K / 4), c4 = (e - r * (K / 4)) * 4;
            const int64_t t = t0 + r;
            const bool valid = t < T;
            cp_async16(dst + sw128_off(r, c4, kTcTok), valid ? m + ((b * T + t) * Hv + h) * K + c4 : m, valid);
        }
        cp_async_commit();
    };
    float mx = 0.0f;
    int64_t cur = -1;       // (b, h) whose S_in^T is staged
    uint32_t phase = 0;
    bool all_ok = true;
    if (i0 < i1) issue_a(i0, 0);
    for (int64_t it = i0; it < i1; ++it) {
        const int buf = static_cast<int>((it - i0) & 1);
        const int64_t bh = it / tiles, t0 = (it - bh * tiles) * kTcTok;
        const int64_t b = bh / Hv, h = bh - b * Hv;
        if (bh != cur) {    // stage B = S_in[b,h]^T, TF32
            cur = bh;
            const float* Sb = S_in + bh * K * V;
            for (int e = threadIdx.x; e < K * V / 4; e += NT) {
                const int i = e / (V / 4), j4 = (e - i * (V / 4)) * 4;
                const float4 v = *reinterpret_cast<const float4*>(Sb + static_cast<int64_t>(i) * V + j4);
                *reinterpret_cast<float*>(sm + L::Bm + sw128_off(j4 + 0, i, V)) = tf32_rn(v.x);
                *reinterpret_cast<float*>(sm + L::Bm + sw128_off(j4 + 1, i, V)) = tf32_rn(v.y);
                *reinterpret_cast<float*>(sm + L::Bm + sw128_off(j4 + 2, i, V)) = tf32_rn(v.z);
                *reinterpret_cast<float*>(sm + L::Bm + sw128_off(j4 + 3, i, V)) = tf32_rn(v.w);
            }
        }
        // the next item's rows go into the other buffer (its last reader, the
        // previous item's MMAs, has completed)
        if (it + 1 < i1) issue_a(it + 1, buf ^ 1);
        else cp_async_commit();
        cp_async_wait<1>();
        {   // round this thread's own chunks of the current buffer to TF32
            uint8_t* a = sm + L::A + buf * L::A_BYTES;
#pragma unroll
            for (int u = 0; u < CPT; ++u) {
                const int e = u * NT + threadIdx.x;
                const int r = e / (K / 4), c4 = (e - r * (K / 4)) * 4;
                float4* p = reinterpret_cast<float4*>(a + sw128_off(r, c4, kTcTok));
                const float4 v = *p;
                *p = make_float4(tf32_rn(v.x), tf32_rn(v.y), tf32_rn(v.z), tf32_rn(v.w));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (threadIdx.x == 0) {
            const uint32_t a = smem_u32(sm + L::A + buf * L::A_BYTES), bb = smem_u32(sm + L::Bm);
#pragma unroll
            for (int j = 0; j < K / 8; ++j)
                mma_tf32_ss(tmem, sdesc_kmajor_sw128(a + (j >> 2) * kTcTok * 128 + (j & 3) * 32),
                            sdesc_kmajor_sw128(bb + (j >> 2) * V * 128 + (j & 3) * 32), IDESC, j > 0 ? 1u : 0u);
            mma_commit(bar);
        }
        // o of this item in the coalesced mapping (a warp per 512 bytes of rows), loaded
        // while the MMAs run: chunk e = u NT + tid is row e / (V/4), 16-byte chunk e % (V/4)
        constexpr int PCH = kTcTok * (V / 4) / NT;
        float4 ov[PCH];
#pragma unroll
        for (int u = 0; u < PCH; ++u) {
            const int e = u * NT + threadIdx.x;
            const int rr = e / (V / 4), cc = e - rr * (V / 4);
            const int64_t tt = t0 + rr;
            ov[u] = tt < T ? *reinterpret_cast<const float4*>(o + ((b * T + tt) * Hv + h) * V + 4 * cc)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const bool ok = __syncthreads_and(mbar_wait(bar, phase, err, kErrTimeoutCorrect));
        if (!ok) {
            all_ok = false;
            break;
        }
        phase ^= 1;
        tc_fence_after();
        {   // D rows (thread = token) into the current A buffer, 16-byte chunks XOR-swizzled by row
            uint32_t x[COLS];
            if constexpr (COLS == 32)
                tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + COLS * cg, x);
            else
                tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(32 * q) << 16) + COLS * cg, x);
            tmem_wait_ld();
            const int r = 32 * q + lane;
            uint8_t* drow = sm + L::A + buf * L::A_BYTES + r * V * 4;
#pragma unroll
            for (int c = 0; c < COLS / 4; ++c) {
                const int chunk = (COLS * cg) / 4 + c;
                *reinterpret_cast<uint4*>(drow + ((chunk ^ (r & 7)) << 4)) =
                    make_uint4(x[4 * c + 0], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
            }
        }
        tc_fence_before();
        __syncthreads();
#pragma unroll
        for (int u = 0; u < PCH; ++u) {
            const int e = u * NT + threadIdx.x;
            const int rr = e / (V / 4), cc = e - rr * (V / 4);
            const int64_t tt = t0 + rr;
            if (tt < T) {
                const float4 d = *reinterpret_cast<const float4*>(sm + L::A + buf * L::A_BYTES + rr * V * 4 +
                                                                  ((cc ^ (rr & 7)) << 4));
                float4 y = ov[u];
                y.x += d.x;
                y.y += d.y;
                y.z += d.z;
                y.w += d.w;
                *reinterpret_cast<float4*>(o + ((b * T + tt) * Hv + h) * V + 4 * cc) = y;
                mx = fmaxf(mx, fmaxf(fmaxf(fabsf(y.x), fabsf(y.y)), fmaxf(fabsf(y.z), fabsf(y.w))));
            }
        }
        __syncthreads();    // the D tile read and B free before the next item
    }
    cp_async_wait<0>();
    if (o_amax) {
        __shared__ unsigned int wmax[NT / 32];
        const unsigned int wm = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
        if (lane == 0) wmax[warp] = wm;
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned int bm = wmax[0];
#pragma unroll
            for (int i = 1; i < NT / 32; ++i) bm = bm > wmax[i] ? bm : wmax[i];
            atomicMax(o_amax, bm);
        }
    }
    // after an expired wait, wait once more (bounded) for the MMAs in flight before TMEM is released
    if (!all_ok && threadIdx.x == 0) mbar_wait(bar, phase, err, kErrTimeoutCorrect);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, V);
    }
}

template <int K, int V>
nvfp4_status launch_correct_tc(const float* m, const float* S_in, float* o, int B, int64_t T, int Hv,
                               unsigned int* o_amax, cudaStream_t st) {
    constexpr int smem = static_cast<int>(CorrTcLayout<K, V>::BYTES);
    static PerDeviceOnce attr_once;
    const nvfp4_status s =
        smem_limit_once(attr_once, scan_correct_tc_kernel<K, V>, smem, "cudaFuncSetAttribute(correct tc)");
    if (s != NVFP4_OK) return s;
    unsigned int* err = device_error_word();
    if (!err) return fail(NVFP4_ERR_CUDA, "device error word unavailable");
    const int64_t n_items = static_cast<int64_t>(B) * Hv * ((T + kTcTok - 1) / kTcTok);
    const int64_t slots = num_sms();
    const int per_cta = static_cast<int>((n_items + slots - 1) / slots);
    const unsigned grid = static_cast<unsigned>((n_items + per_cta - 1) / per_cta);
    const cudaError_t e = launch_pdl(scan_correct_tc_kernel<K, V>, dim3(grid), dim3(512), smem, st, m, S_in, o, T,
                                     Hv, n_items, per_cta, o_amax, err);
    if (e != cudaSuccess) return cuda_fail(e, "scan correct launch");
    return NVFP4_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const char* pa = static_cast<const char*>(a);
    const char* pb = static_cast<const char*>(b);
    return a && b && pa < pb + nb && pb < pa + na;
}

}  // namespace

nvfp4_status identity_fill_launch(float* P, int64_t n_mat, int K, float* zero_row, int64_t n_zero,
                                  cudaStream_t st) {
    const int64_t total = n_mat * K * K;
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((total + 255) / 256, int64_t(num_sms()) * 8));
    const cudaError_t e = launch_pdl(identity_fill_kernel, dim3(blocks), dim3(256), 0, st, P, n_mat, K, zero_row, n_zero);
    if (e != cudaSuccess) return cuda_fail(e, "identity fill launch");
    return NVFP4_OK;
}

size_t transition_workspace_bytes(int B, int64_t T, const gdn_dims& d, int algo) {
    gdn_dims dk = d;
    dk.V = d.K;
    return round_up(scan_workspace_bytes(B, T, dk, algo)) + round_up(static_cast<size_t>(d.Hv) * d.K * 4);
}

}  // namespace nvg

extern "C" size_t gdn_scan_transition_workspace_size(int32_t B, int64_t T, const gdn_dims* dims, int32_t algo) {
    if (!dims || nvg::validate_dims(dims) != NVFP4_OK || B < 1 || T < 1) return 0;
    return nvg::transition_workspace_bytes(B, T, *dims, algo);
}

extern "C" nvfp4_status gdn_scan_transition(const float* q_hat, const float* k_hat, const float* g, const float* beta,
                                            int32_t B, int64_t T, const gdn_dims* dims, float scale, int32_t form,
                                            int32_t algo, float* P, float* qmap, void* workspace,
                                            size_t workspace_bytes, nvfp4_stream_t stream) {
    using namespace nvg;
    nvfp4_status s = validate_dims(dims);
    if (s != NVFP4_OK) return s;
    if (!q_hat || !k_hat || !g || !beta || !P || !qmap) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
    if (B < 1 || T < 1) return fail(NVFP4_ERR_INVALID_ARG, "B and T must be >= 1");
    if (form != GDN_FORM_PAGES && form != GDN_FORM_STANDARD) return fail(NVFP4_ERR_INVALID_ARG, "bad form");
    if (algo != GDN_SCAN_AUTO && algo != GDN_SCAN_RECURRENT && algo != GDN_SCAN_CHUNKED)
        return fail(NVFP4_ERR_INVALID_ARG, "bad algo");
    if (static_cast<int64_t>(B) * T > (int64_t(1) << 31)) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "B*T too large");
    if (!aligned16(q_hat) || !aligned16(k_hat) || !aligned16(P) || !aligned16(qmap))
        return fail(NVFP4_ERR_MISALIGNED, "q_hat, k_hat, P, qmap must be 16-byte aligned");
    const size_t need = transition_workspace_bytes(B, T, *dims, algo);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return fail(NVFP4_ERR_WORKSPACE, "transition workspace missing, too small or not 256-byte aligned");
    const size_t p_bytes = static_cast<size_t>(B) * dims->Hv * dims->K * dims->K * 4;
    const size_t m_bytes = static_cast<size_t>(B) * T * dims->Hv * dims->K * 4;
    if (overlaps(P, p_bytes, qmap, m_bytes) || overlaps(P, p_bytes, workspace, need) ||
        overlaps(qmap, m_bytes, workspace, need))
        return fail(NVFP4_ERR_INVALID_ARG, "P, qmap and the workspace must not overlap");
    gdn_dims dk = *dims;
    dk.V = dims->K;
    const size_t zero_off = round_up(scan_workspace_bytes(B, T, dk, algo));
    float* zero_row = reinterpret_cast<float*>(static_cast<char*>(workspace) + zero_off);
    const cudaStream_t st = as_stream(stream);
    if ((s = identity_fill_launch(P, static_cast<int64_t>(B) * dims->Hv, dims->K, zero_row,
                                  static_cast<int64_t>(dims->Hv) * dims->K, st)) != NVFP4_OK)
        return s;
    // v = 0 (every token reads the same zero row: row stride 0), state P in place
    return scan_launch(q_hat, k_hat, zero_row, 0, g, beta, B, T, dk, scale, form, algo, P, P, qmap, workspace, st,
                       nullptr, static_cast<int64_t>(dims->Hk) * dims->K, 0);
}

extern "C" nvfp4_status gdn_state_combine(const float* P, const float* S_loc, const float* S_in, float* S_out,
                                          int32_t m, int64_t n, int32_t K, int32_t V, nvfp4_stream_t stream) {
    using namespace nvg;
    if (!S_out || !P) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
    if (m < 1 || n < 1) return fail(NVFP4_ERR_INVALID_ARG, "m and n must be >= 1");
    if ((K != 32 && K != 64 && K != 128) || V < 32 || V % 32 || V / 32 > 65535)
        return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K must be 32, 64 or 128 and V a multiple of 32");
    if (n > 2147483647) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "n too large");
    if (!aligned16(P)) return fail(NVFP4_ERR_MISALIGNED, "P must be 16-byte aligned");
    const size_t s_bytes = static_cast<size_t>(n) * K * V * 4;
    const size_t p_bytes = static_cast<size_t>(m) * n * K * K * 4;
    if (overlaps(S_out, s_bytes, P, p_bytes)) return fail(NVFP4_ERR_INVALID_ARG, "S_out must not overlap P");
    if (S_in && S_in != S_out && overlaps(S_out, s_bytes, S_in, s_bytes))
        return fail(NVFP4_ERR_INVALID_ARG, "S_out must be S_in or not overlap it");
    const float* last = S_loc ? S_loc + static_cast<int64_t>(m - 1) * n * K * V : nullptr;
    if (S_loc && S_out != last && overlaps(S_out, s_bytes, S_loc, static_cast<size_t>(m) * s_bytes))
        return fail(NVFP4_ERR_INVALID_ARG, "S_out must be the last S_loc or not overlap S_loc");
    const cudaStream_t st = as_stream(stream);
    if (K == 128) return launch_chain<128>(P, S_loc, S_in, S_out, m, n, V, st);
    if (K == 64) return launch_chain<64>(P, S_loc, S_in, S_out, m, n, V, st);
    return launch_chain<32>(P, S_loc, S_in, S_out, m, n, V, st);
}

extern "C" nvfp4_status gdn_scan_correct(const float* qmap, const float* S_in, float* o, int32_t B, int64_t T,
                                         int32_t Hv, int32_t K, int32_t V, unsigned int* o_amax,
                                         nvfp4_stream_t stream) {
    using namespace nvg;
    if (!qmap || !S_in || !o) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
    if (B < 1 || T < 1 || Hv < 1) return fail(NVFP4_ERR_INVALID_ARG, "B, T and Hv must be >= 1");
    if ((K != 64 && K != 128) || (V != 64 && V != 128))
        return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "head dims K, V must be 64 or 128");
    if (B > 65535 || Hv > 65535 || static_cast<int64_t>(B) * T > (int64_t(1) << 31))
        return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "B, Hv or B*T too large");
    if (!aligned16(qmap) || !aligned16(S_in) || !aligned16(o))
        return fail(NVFP4_ERR_MISALIGNED, "qmap, S_in, o must be 16-byte aligned");
    const size_t o_bytes = static_cast<size_t>(B) * T * Hv * V * 4;
    if (overlaps(o, o_bytes, qmap, static_cast<size_t>(B) * T * Hv * K * 4) ||
        overlaps(o, o_bytes, S_in, static_cast<size_t>(B) * Hv * K * V * 4))
        return fail(NVFP4_ERR_INVALID_ARG, "o must not overlap qmap or S_in");
    const cudaStream_t st = as_stream(stream);
    unsigned int* amax = o_amax;
    const char* var = getenv("NVFP4_CORRECT_VARIANT");
    if (var && strcmp(var, "cuda_core") == 0) {
        if (K == 128 && V == 128) return launch_correct<128, 128>(qmap, S_in, o, B, T, Hv, amax, st);
        if (K == 128 && V == 64) return launch_correct<128, 64>(qmap, S_in, o, B, T, Hv, amax, st);
        if (K == 64 && V == 128) return launch_correct<64, 128>(qmap, S_in, o, B, T, Hv, amax, st);
        return launch_correct<64, 64>(qmap, S_in, o, B, T, Hv, amax, st);
    }
    if (K == 128 && V == 128) return launch_correct_tc<128, 128>(qmap, S_in, o, B, T, Hv, amax, st);
    if (K == 128 && V == 64) return launch_correct_tc<128, 64>(qmap, S_in, o, B, T, Hv, amax, st);
    if (K == 64 && V == 128) return launch_correct_tc<64, 128>(qmap, S_in, o, B, T, Hv, amax, st);
    return launch_correct_tc<64, 64>(qmap, S_in, o, B, T, Hv, amax, st);
}
