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
//   gdn_state_combine     S_out = P S_in + S_loc per (sequence, value head);
//   gdn_scan_correct      o_t += S_in^T m_t over a span's tokens, with the
//                         quantiser's amax of the corrected o folded in.
#include <algorithm>

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

// S_out[n] = P[n] S_in[n] + S_loc[n].  One CTA per (n, 32 rows of the output);
// warp w owns rows 4w..4w+3 of the block, lane l the columns l + 32c.  The 32
// rows of P sit in shared memory and are read as broadcasts; the rows of S_in
// are read coalesced (the CTAs of one n share them through L1/L2).
constexpr int kCombRows = 32;
__global__ void __launch_bounds__(256) state_combine_kernel(const float* __restrict__ P,
                                                            const float* S_loc,
                                                            const float* __restrict__ S_in, float* S_out,
                                                            int K, int V) {
    pdl_wait_and_trigger();
    __shared__ float Ps[kCombRows][256];
    const int64_t n = blockIdx.x;
    const int i0 = blockIdx.y * kCombRows;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int VC = V >> 5;
    float acc[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = 0.0f;
    if (S_in) {
        const float* Pn = P + n * K * K;
        for (int e = threadIdx.x; e < kCombRows * K; e += blockDim.x) Ps[e / K][e % K] = Pn[static_cast<int64_t>(i0 + e / K) * K + e % K];
        __syncthreads();
        const float* Sn = S_in + n * K * V;
        for (int l = 0; l < K; ++l) {
            float s[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) s[c] = c < VC ? Sn[static_cast<int64_t>(l) * V + lane + 32 * c] : 0.0f;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float p = Ps[4 * w + r][l];
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(p, s[c], acc[r][c]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t row = n * K * V + static_cast<int64_t>(i0 + 4 * w + r) * V;
#pragma unroll
        for (int c = 0; c < 8; ++c)
            if (c < VC) {
                const int64_t e = row + lane + 32 * c;
                S_out[e] = acc[r][c] + (S_loc ? S_loc[e] : 0.0f);
            }
    }
}

// o[b,t,h,:] += S_in[b,h]^T m[b,t,h,:] over a tile of 64 tokens of one (b, h).
// S_in[b,h] (K x V) and the tile's m rows (64 x K) are staged in shared memory;
// thread (ty, tx) of a 16 x 16 grid owns tokens 4ty..4ty+3 and the columns
// 4tx + 64c .. +3 (c < V/64), so each step over 4 values of k takes 4 + 4 V/64
// 16-byte shared loads for 64 V/64 FMAs.  The largest |o| of the CTA goes into
// the quantiser's amax word with one atomicMax.
constexpr int kCorrTok = 64;
template <int K, int V>
__global__ void __launch_bounds__(256) scan_correct_kernel(const float* __restrict__ m, const float* __restrict__ S_in,
                                                           float* __restrict__ o, int64_t T, int Hv,
                                                           unsigned int* __restrict__ o_amax) {
    pdl_wait_and_trigger();
    constexpr int VC = V / 64;
    extern __shared__ __align__(16) float smem[];
    float* Ss = smem;              // [K][V]
    float* Ms = smem + K * V;      // [kCorrTok][K]
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kCorrTok;
    const int h = blockIdx.y, b = blockIdx.z;
    const float4* S4 = reinterpret_cast<const float4*>(S_in + (static_cast<int64_t>(b) * Hv + h) * K * V);
    for (int e = threadIdx.x; e < K * V / 4; e += 256) reinterpret_cast<float4*>(Ss)[e] = S4[e];
    for (int e = threadIdx.x; e < kCorrTok * K / 4; e += 256) {
        const int r = e / (K / 4), c4 = e % (K / 4);
        const int64_t t = t0 + r;
        reinterpret_cast<float4*>(Ms)[e] =
            t < T ? *reinterpret_cast<const float4*>(m + ((static_cast<int64_t>(b) * T + t) * Hv + h) * K + 4 * c4)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4 * VC];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4 * VC; ++c) acc[r][c] = 0.0f;
#pragma unroll 2
    for (int kk = 0; kk < K; kk += 4) {
        float4 a[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) a[r] = *reinterpret_cast<const float4*>(Ms + (4 * ty + r) * K + kk);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4 s[VC];
#pragma unroll
            for (int c = 0; c < VC; ++c) s[c] = *reinterpret_cast<const float4*>(Ss + (kk + q) * V + 4 * tx + 64 * c);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float av = q == 0 ? a[r].x : q == 1 ? a[r].y : q == 2 ? a[r].z : a[r].w;
#pragma unroll
                for (int c = 0; c < VC; ++c) {
                    acc[r][4 * c + 0] = fmaf(av, s[c].x, acc[r][4 * c + 0]);
                    acc[r][4 * c + 1] = fmaf(av, s[c].y, acc[r][4 * c + 1]);
                    acc[r][4 * c + 2] = fmaf(av, s[c].z, acc[r][4 * c + 2]);
                    acc[r][4 * c + 3] = fmaf(av, s[c].w, acc[r][4 * c + 3]);
                }
            }
        }
    }
    float mx = 0.0f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t t = t0 + 4 * ty + r;
        if (t < T) {
            float* orow = o + ((static_cast<int64_t>(b) * T + t) * Hv + h) * V;
#pragma unroll
            for (int c = 0; c < VC; ++c) {
                float4* p = reinterpret_cast<float4*>(orow + 4 * tx + 64 * c);
                float4 x = *p;
                x.x += acc[r][4 * c + 0];
                x.y += acc[r][4 * c + 1];
                x.z += acc[r][4 * c + 2];
                x.w += acc[r][4 * c + 3];
                *p = x;
                mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
            }
        }
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
    constexpr int smem = (K * V + kCorrTok * K) * 4;
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(scan_correct_kernel<K, V>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(correct)");
        attr_done[dev] = true;
    }
    const dim3 grid(static_cast<unsigned>((T + kCorrTok - 1) / kCorrTok), Hv, B);
    const cudaError_t e = launch_pdl(scan_correct_kernel<K, V>, grid, dim3(256), smem, st, m, S_in, o, T, Hv, o_amax);
    if (e != cudaSuccess) return cuda_fail(e, "scan correct launch");
    return NVFP4_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const char* pa = static_cast<const char*>(a);
    const char* pb = static_cast<const char*>(b);
    return a && b && pa < pb + nb && pb < pa + na;
}

}  // namespace

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
    const int64_t n_mat = static_cast<int64_t>(B) * dims->Hv;
    const int64_t total = n_mat * dims->K * dims->K;
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((total + 255) / 256, int64_t(num_sms()) * 8));
    const cudaError_t e = launch_pdl(identity_fill_kernel, dim3(blocks), dim3(256), 0, st, P, n_mat, dims->K, zero_row,
                                     static_cast<int64_t>(dims->Hv) * dims->K);
    if (e != cudaSuccess) return cuda_fail(e, "identity fill launch");
    // v = 0 (every token reads the same zero row: row stride 0), state P in place
    return scan_launch(q_hat, k_hat, zero_row, 0, g, beta, B, T, dk, scale, form, algo, P, P, qmap, workspace, st,
                       nullptr, static_cast<int64_t>(dims->Hk) * dims->K, 0);
}

extern "C" nvfp4_status gdn_state_combine(const float* P, const float* S_loc, const float* S_in, float* S_out,
                                          int64_t n, int32_t K, int32_t V, nvfp4_stream_t stream) {
    using namespace nvg;
    if (!S_out || (S_in && !P)) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
    if (n < 1) return fail(NVFP4_ERR_INVALID_ARG, "n must be >= 1");
    if (K < 32 || K > 256 || K % 32 || V < 32 || V > 256 || V % 32)
        return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K and V must be multiples of 32 in [32, 256]");
    if (n > 2147483647) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "n too large");
    const size_t s_bytes = static_cast<size_t>(n) * K * V * 4;
    const size_t p_bytes = static_cast<size_t>(n) * K * K * 4;
    if (overlaps(S_out, s_bytes, S_in, s_bytes) || overlaps(S_out, s_bytes, P, p_bytes))
        return fail(NVFP4_ERR_INVALID_ARG, "S_out must not overlap P or S_in");
    if (S_loc && S_loc != S_out && overlaps(S_out, s_bytes, S_loc, s_bytes))
        return fail(NVFP4_ERR_INVALID_ARG, "S_out must be S_loc or not overlap it");
    const cudaError_t e = launch_pdl(state_combine_kernel, dim3(static_cast<unsigned>(n), K / kCombRows), dim3(256), 0,
                                     as_stream(stream), P, S_loc, S_in, S_out, K, V);
    if (e != cudaSuccess) return cuda_fail(e, "state combine launch");
    return NVFP4_OK;
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
    if (K == 128 && V == 128) return launch_correct<128, 128>(qmap, S_in, o, B, T, Hv, amax, st);
    if (K == 128 && V == 64) return launch_correct<128, 64>(qmap, S_in, o, B, T, Hv, amax, st);
    if (K == 64 && V == 128) return launch_correct<64, 128>(qmap, S_in, o, B, T, Hv, amax, st);
    return launch_correct<64, 64>(qmap, S_in, o, B, T, Hv, amax, st);
}
