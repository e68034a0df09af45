// gates.cu -- gate parameterisation (Eq.(1) of the review page of "Why Gated
// DeltaNet Survives 4-Bit Quantization", paper sec.2) and per-head q/k L2
// normalisation, read straight from the fused projection's column slices.
//
//   g     = -exp(A_log) * softplus(a + dt_bias)   (log of alpha, alpha = e^g in (0,1))
//   beta  = sigmoid(b)
//   q_hat = q / sqrt(sum q^2 + 1e-6), same for k
//
// Element-wise and HBM-bound: one warp per (token, head) row for the
// normalisation (coalesced 16-byte loads), one thread per (token, value head)
// for the gates.
//
// Also the optional output gate before out_proj (the pages name z as moving the
// output y, review page Table 3 discussion, and keep the norms unquantised,
// "Minima" section; the formula is this library's reading, the usual gated
// RMSNorm): out = o / sqrt(mean(o^2) + 1e-6) * w * SiLU(z) per (token, value
// head), warps walking rows, the |out| maximum folded into an amax word for the
// quantiser that follows.
#include <type_traits>

#include "common.cuh"

namespace nvg {

namespace {

template <int D>
__global__ void __launch_bounds__(256) l2norm_kernel(const float* __restrict__ proj, int64_t ld, int64_t n_tokens,
                                                     int Hk, float* __restrict__ q_hat, float* __restrict__ k_hat) {
    pdl_wait_and_trigger();
    constexpr int PER_LANE = D / 32;  // 2 or 4 contiguous floats per lane
    const int64_t gw = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t rows = n_tokens * Hk * 2;
    if (gw >= rows) return;
    const int which = static_cast<int>(gw % 2);  // 0 = q, 1 = k
    const int64_t th = gw / 2;
    const int64_t t = th / Hk;
    const int h = static_cast<int>(th - t * Hk);
    const float* src = proj + t * ld + static_cast<int64_t>(which) * Hk * D + static_cast<int64_t>(h) * D + lane * PER_LANE;
    float v[PER_LANE];
    if constexpr (PER_LANE == 4) {
        const float4 u = *reinterpret_cast<const float4*>(src);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    } else {
        const float2 u = *reinterpret_cast<const float2*>(src);
        v[0] = u.x; v[1] = u.y;
    }
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) ss = fmaf(v[i], v[i], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss + 1e-6f);
    float* dst = (which == 0 ? q_hat : k_hat) + th * D + lane * PER_LANE;
    if constexpr (PER_LANE == 4) {
        *reinterpret_cast<float4*>(dst) = make_float4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
    } else {
        *reinterpret_cast<float2*>(dst) = make_float2(v[0] * inv, v[1] * inv);
    }
}

__global__ void __launch_bounds__(256) gate_kernel(const float* __restrict__ proj, int64_t ld, int64_t n_tokens, int Hv,
                                                   int64_t col_a, int64_t col_b, const float* __restrict__ A_log,
                                                   const float* __restrict__ dt_bias, float* __restrict__ g,
                                                   float* __restrict__ beta) {
    pdl_wait_and_trigger();
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= n_tokens * Hv) return;
    const int64_t t = i / Hv;
    const int h = static_cast<int>(i - t * Hv);
    const float a = proj[t * ld + col_a + h];
    const float b = proj[t * ld + col_b + h];
    const float u = a + dt_bias[h];
    const float sp = fmaxf(u, 0.0f) + log1pf(expf(-fabsf(u)));
    g[i] = -expf(A_log[h]) * sp;
    beta[i] = 1.0f / (1.0f + expf(-b));
}

// Each warp walks (token, value head) rows of V values, V/32 per lane, in a
// grid-stride loop; one atomicMax per CTA folds the |out| maximum into the amax
// word (one per row would serialise on that word).
template <int V>
__global__ void __launch_bounds__(256) output_gate_kernel(const float* o, const float* __restrict__ z, int64_t ld_z,
                                                          const float* __restrict__ w, int64_t n_tokens, int Hv,
                                                          float* out, unsigned int* __restrict__ amax_word) {
    pdl_wait_and_trigger();
    constexpr int PL = V / 32;
    using VecT = typename std::conditional<PL == 4, float4, float2>::type;
    const int lane = threadIdx.x & 31;
    const int64_t rows = n_tokens * Hv;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    float wv[PL];
    {
        const VecT c = *reinterpret_cast<const VecT*>(w + lane * PL);
        memcpy(wv, &c, sizeof(wv));
    }
    float m = 0.0f;
    // two rows per iteration, both rows' loads issued before either is used
    constexpr int R = 2;
    for (int64_t row0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; row0 < rows;
         row0 += R * nwarps) {
        float ov[R][PL], zv[R][PL];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t row = row0 + r * nwarps;
            VecT a{}, b{};
            if (row < rows) {
                const int64_t t = row / Hv;
                const int h = static_cast<int>(row - t * Hv);
                a = *reinterpret_cast<const VecT*>(o + row * V + lane * PL);
                b = *reinterpret_cast<const VecT*>(z + t * ld_z + static_cast<int64_t>(h) * V + lane * PL);
            }
            memcpy(ov[r], &a, sizeof(ov[r]));
            memcpy(zv[r], &b, sizeof(zv[r]));
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t row = row0 + r * nwarps;
            float ss = 0.0f;
#pragma unroll
            for (int i = 0; i < PL; ++i) ss = fmaf(ov[r][i], ov[r][i], ss);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float inv_rms = 1.0f / sqrtf(ss / static_cast<float>(V) + 1e-6f);
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const float silu = zv[r][i] / (1.0f + expf(-zv[r][i]));
                ov[r][i] = ov[r][i] * inv_rms * wv[i] * silu;
                m = fmaxf(m, fabsf(ov[r][i]));
            }
            if (row < rows) {
                VecT res;
                memcpy(&res, ov[r], sizeof(ov[r]));
                *reinterpret_cast<VecT*>(out + row * V + lane * PL) = res;
            }
        }
    }
    if (amax_word) {
        __shared__ unsigned int warp_max[8];
        const unsigned int mb = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
        if (lane == 0) warp_max[threadIdx.x >> 5] = mb;
        __syncthreads();
        if (threadIdx.x < 32) {
            unsigned int v = threadIdx.x < (blockDim.x >> 5) ? warp_max[threadIdx.x] : 0u;
            v = __reduce_max_sync(0xffffffffu, v);
            if (threadIdx.x == 0) atomicMax(amax_word, v);
        }
    }
}

}  // namespace

nvfp4_status validate_dims(const gdn_dims* d) {
    if (!d) return fail(NVFP4_ERR_INVALID_ARG, "dims is null");
    if (d->Hk < 1 || d->Hv < 1 || d->Hv % d->Hk) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "Hv must be a multiple of Hk");
    if ((d->K != 64 && d->K != 128) || (d->V != 64 && d->V != 128))
        return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "head dims K, V must be 64 or 128");
    return NVFP4_OK;
}

nvfp4_status gate_only_launch(const float* proj, int64_t ld, int64_t n, const gdn_dims& d, const float* A_log,
                              const float* dt_bias, float* g, float* beta, cudaStream_t st);

// q_hat, k_hat from rows whose first 2 Hk K columns are q | k (row stride ld).
nvfp4_status l2norm_launch(const float* proj, int64_t ld, int64_t n, const gdn_dims& d, float* q_hat, float* k_hat,
                           cudaStream_t st) {
    const int64_t warps = n * d.Hk * 2;
    const unsigned blocks_n = static_cast<unsigned>((warps * 32 + 255) / 256);
    cudaError_t e;
    if (d.K == 128)
        e = launch_pdl(l2norm_kernel<128>, dim3(blocks_n), dim3(256), 0, st, proj, ld, n, d.Hk, q_hat, k_hat);
    else
        e = launch_pdl(l2norm_kernel<64>, dim3(blocks_n), dim3(256), 0, st, proj, ld, n, d.Hk, q_hat, k_hat);
    if (e != cudaSuccess) return cuda_fail(e, "l2norm launch");
    return NVFP4_OK;
}

nvfp4_status gates_launch(const float* proj, int64_t ld, int64_t n, const gdn_dims& d, const float* A_log,
                          const float* dt_bias, float* q_hat, float* k_hat, float* g, float* beta, cudaStream_t st) {
    nvfp4_status s = l2norm_launch(proj, ld, n, d, q_hat, k_hat, st);
    if (s != NVFP4_OK) return s;
    return gate_only_launch(proj, ld, n, d, A_log, dt_bias, g, beta, st);
}

// g and beta only (the chunked scan can normalise q, k itself while loading them).
nvfp4_status gate_only_launch(const float* proj, int64_t ld, int64_t n, const gdn_dims& d, const float* A_log,
                              const float* dt_bias, float* g, float* beta, cudaStream_t st) {
    const int64_t col_a = 2ll * d.Hk * d.K + 2ll * d.Hv * d.V;
    const unsigned blocks_g = static_cast<unsigned>((n * d.Hv + 255) / 256);
    const cudaError_t e = launch_pdl(gate_kernel, dim3(blocks_g), dim3(256), 0, st, proj, ld, n, d.Hv, col_a,
                                     col_a + d.Hv, A_log, dt_bias, g, beta);
    if (e != cudaSuccess) return cuda_fail(e, "gates launch");
    return NVFP4_OK;
}

nvfp4_status output_gate_launch(const float* o, const float* z, int64_t ld_z, const float* w, int64_t n, int Hv, int V,
                                float* out, unsigned int* amax_word, cudaStream_t st) {
    const int64_t rows = n * Hv;
    int64_t blocks64 = (rows + 7) / 8;                         // one row per warp at most
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;  // resident CTAs of 8 warps
    if (blocks64 > cap) blocks64 = cap;
    const unsigned blocks = static_cast<unsigned>(blocks64);
    const cudaError_t e =
        V == 128 ? launch_pdl(output_gate_kernel<128>, dim3(blocks), dim3(256), 0, st, o, z, ld_z, w, n, Hv, out, amax_word)
                 : launch_pdl(output_gate_kernel<64>, dim3(blocks), dim3(256), 0, st, o, z, ld_z, w, n, Hv, out, amax_word);
    if (e != cudaSuccess) return cuda_fail(e, "output gate launch");
    return NVFP4_OK;
}

}  // namespace nvg

extern "C" nvfp4_status gdn_gates(const float* proj, int64_t ld_proj, int64_t n_tokens, const gdn_dims* dims,
                                  const float* A_log, const float* dt_bias, float* q_hat, float* k_hat, float* g,
                                  float* beta, nvfp4_stream_t stream) {
    using namespace nvg;
    nvfp4_status s = validate_dims(dims);
    if (s != NVFP4_OK) return s;
    if (!proj || !A_log || !dt_bias || !q_hat || !k_hat || !g || !beta)
        return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
    if (n_tokens < 1) return fail(NVFP4_ERR_INVALID_ARG, "n_tokens < 1");
    const int64_t n_in = 2ll * dims->Hk * dims->K + 2ll * dims->Hv * dims->V + 2ll * dims->Hv;
    if (ld_proj < n_in) return fail(NVFP4_ERR_INVALID_ARG, "ld_proj smaller than the fused projection width");
    if (!aligned16(proj) || ld_proj % 4 || !aligned16(q_hat) || !aligned16(k_hat))
        return fail(NVFP4_ERR_MISALIGNED, "proj / q_hat / k_hat must be 16-byte aligned, ld_proj % 4 == 0");
    return gates_launch(proj, ld_proj, n_tokens, *dims, A_log, dt_bias, q_hat, k_hat, g, beta, as_stream(stream));
}

extern "C" nvfp4_status gdn_output_gate(const float* o, const float* z, int64_t ld_z, const float* w, int64_t n_tokens,
                                        int32_t Hv, int32_t V, float* out, unsigned int* amax_word,
                                        nvfp4_stream_t stream) {
    using namespace nvg;
    if (!o || !z || !w || !out) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
    if (n_tokens < 1 || Hv < 1) return fail(NVFP4_ERR_INVALID_ARG, "n_tokens and Hv must be >= 1");
    if (V != 64 && V != 128) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "V must be 64 or 128");
    if (ld_z < static_cast<int64_t>(Hv) * V) return fail(NVFP4_ERR_INVALID_ARG, "ld_z smaller than Hv*V");
    if (!aligned16(o) || !aligned16(z) || !aligned16(w) || !aligned16(out) || ld_z % 4)
        return fail(NVFP4_ERR_MISALIGNED, "o / z / w / out must be 16-byte aligned, ld_z % 4 == 0");
    return output_gate_launch(o, z, ld_z, w, n_tokens, Hv, V, out, amax_word, as_stream(stream));
}
