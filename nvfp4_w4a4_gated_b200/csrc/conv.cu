// conv.cu -- optional short causal convolution on the q|k|v channels of the
// fused projection.  The review page of "Why Gated DeltaNet Survives 4-Bit
// Quantization" lists convolutions among the layers kept unquantised ("Minima"
// section) and says nothing more; this library reads it as the usual Gated
// DeltaNet short convolution, per channel c and token t:
//
//   out_t[c] = SiLU(sum_{j < W} w[c][j] * x_{t-W+1+j}[c]),   SiLU(u) = u / (1 + e^-u)
//
// with the inputs before a call's first token taken from a carried state (the
// previous W-1 inputs of the sequence, zero when absent).
//
// HBM-bound.  When the channel count and the row strides allow 16-byte access,
// each thread takes four channels over a block of 16 tokens with all of the
// block's inputs loaded before any is used; otherwise one thread per channel
// slides a window of W inputs over 32 tokens.  A warp's loads and stores are
// consecutive channels (coalesced).  A second small kernel writes the new state
// after the first has read the old one, so the state may be updated in place.
#include "common.cuh"

namespace nvg {

namespace {

constexpr int kConvTokens = 32;    // tokens per CTA
constexpr int kConvThreads = 128;  // channels per CTA

template <int W>
__global__ void __launch_bounds__(kConvThreads) short_conv_kernel(const float* __restrict__ x, int64_t ld_x, int64_t T,
                                                                  int C, const float* __restrict__ w,
                                                                  const float* __restrict__ state_in,
                                                                  float* __restrict__ out, int64_t ld_out) {
    pdl_wait_and_trigger();
    const int c = blockIdx.x * kConvThreads + threadIdx.x;
    const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kConvTokens;
    const int b = blockIdx.z;
    if (c >= C || t0 >= T) return;
    float tap[W];
#pragma unroll
    for (int j = 0; j < W; ++j) tap[j] = w[static_cast<int64_t>(c) * W + j];
    // window[j] = input at token t - (W-1) + j; preload the W-1 inputs before t0
    float win[W];
#pragma unroll
    for (int j = 0; j < W - 1; ++j) {
        const int64_t u = t0 - (W - 1) + j;
        if (u >= 0)
            win[j] = x[(static_cast<int64_t>(b) * T + u) * ld_x + c];
        else
            win[j] = state_in ? state_in[(static_cast<int64_t>(b) * C + c) * (W - 1) + (u + (W - 1))] : 0.0f;
    }
    const int64_t t1 = t0 + kConvTokens < T ? t0 + kConvTokens : T;
    for (int64_t t = t0; t < t1; ++t) {
        win[W - 1] = x[(static_cast<int64_t>(b) * T + t) * ld_x + c];
        float acc = 0.0f;
#pragma unroll
        for (int j = 0; j < W; ++j) acc = fmaf(tap[j], win[j], acc);
        out[(static_cast<int64_t>(b) * T + t) * ld_out + c] = acc / (1.0f + expf(-acc));
#pragma unroll
        for (int j = 0; j < W - 1; ++j) win[j] = win[j + 1];
    }
}

// Four channels per thread (16-byte loads and stores) over a block of kConvTokens4
// tokens, whose inputs are all loaded before any is used.  Needs C, ld_x and
// ld_out multiples of 4 and 16-byte aligned x, out.
constexpr int kConvTokens4 = 16;
template <int W>
__global__ void __launch_bounds__(kConvThreads) short_conv4_kernel(const float* __restrict__ x, int64_t ld_x, int64_t T,
                                                                   int C, const float* __restrict__ w,
                                                                   const float* __restrict__ state_in,
                                                                   float* __restrict__ out, int64_t ld_out) {
    pdl_wait_and_trigger();
    const int c0 = (blockIdx.x * kConvThreads + threadIdx.x) * 4;
    const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kConvTokens4;
    const int b = blockIdx.z;
    if (c0 >= C || t0 >= T) return;
    const int n = static_cast<int>(T - t0 < kConvTokens4 ? T - t0 : kConvTokens4);
    float tap[4][W];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int j = 0; j < W; ++j) tap[k][j] = w[static_cast<int64_t>(c0 + k) * W + j];
    float4 in[W - 1 + kConvTokens4];
#pragma unroll
    for (int j = 0; j < W - 1; ++j) {
        const int64_t u = t0 - (W - 1) + j;
        if (u >= 0) {
            in[j] = *reinterpret_cast<const float4*>(x + (static_cast<int64_t>(b) * T + u) * ld_x + c0);
        } else if (state_in) {
            const float* sp = state_in + static_cast<int64_t>(b) * C * (W - 1) + (u + (W - 1));
            in[j] = make_float4(sp[static_cast<int64_t>(c0) * (W - 1)], sp[static_cast<int64_t>(c0 + 1) * (W - 1)],
                                sp[static_cast<int64_t>(c0 + 2) * (W - 1)], sp[static_cast<int64_t>(c0 + 3) * (W - 1)]);
        } else {
            in[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
#pragma unroll
    for (int i = 0; i < kConvTokens4; ++i)
        in[W - 1 + i] = i < n ? *reinterpret_cast<const float4*>(x + (static_cast<int64_t>(b) * T + t0 + i) * ld_x + c0)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kConvTokens4; ++i) {
        if (i < n) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < W; ++j) {
                const float4 v = in[i + j];
                acc[0] = fmaf(tap[0][j], v.x, acc[0]);
                acc[1] = fmaf(tap[1][j], v.y, acc[1]);
                acc[2] = fmaf(tap[2][j], v.z, acc[2]);
                acc[3] = fmaf(tap[3][j], v.w, acc[3]);
            }
            *reinterpret_cast<float4*>(out + (static_cast<int64_t>(b) * T + t0 + i) * ld_out + c0) =
                make_float4(acc[0] / (1.0f + expf(-acc[0])), acc[1] / (1.0f + expf(-acc[1])),
                            acc[2] / (1.0f + expf(-acc[2])), acc[3] / (1.0f + expf(-acc[3])));
        }
    }
}

// New state: the last W-1 inputs of each sequence (some from the old state when
// T < W-1).  Each thread reads all it needs before writing, so in place is safe.
template <int W>
__global__ void __launch_bounds__(kConvThreads) short_conv_state_kernel(const float* __restrict__ x, int64_t ld_x,
                                                                        int64_t T, int C, const float* state_in,
                                                                        float* state_out) {
    pdl_wait_and_trigger();
    const int c = blockIdx.x * kConvThreads + threadIdx.x;
    const int b = blockIdx.y;
    if (c >= C) return;
    float v[W - 1];
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
        const int64_t u = T - (W - 1) + i;
        if (u >= 0)
            v[i] = x[(static_cast<int64_t>(b) * T + u) * ld_x + c];
        else
            v[i] = state_in ? state_in[(static_cast<int64_t>(b) * C + c) * (W - 1) + (u + (W - 1))] : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < W - 1; ++i) state_out[(static_cast<int64_t>(b) * C + c) * (W - 1) + i] = v[i];
}

template <int W>
nvfp4_status launch_conv(const float* x, int64_t ld_x, int B, int64_t T, int C, const float* w, const float* state_in,
                         float* state_out, float* out, int64_t ld_out, cudaStream_t st) {
    cudaError_t e;
    if (C % 4 == 0 && ld_x % 4 == 0 && ld_out % 4 == 0 && aligned16(x) && aligned16(out)) {
        const dim3 grid((C / 4 + kConvThreads - 1) / kConvThreads,
                        static_cast<unsigned>((T + kConvTokens4 - 1) / kConvTokens4), B);
        e = launch_pdl(short_conv4_kernel<W>, grid, dim3(kConvThreads), 0, st, x, ld_x, T, C, w, state_in, out, ld_out);
    } else {
        const dim3 grid((C + kConvThreads - 1) / kConvThreads,
                        static_cast<unsigned>((T + kConvTokens - 1) / kConvTokens), B);
        e = launch_pdl(short_conv_kernel<W>, grid, dim3(kConvThreads), 0, st, x, ld_x, T, C, w, state_in, out, ld_out);
    }
    if (e != cudaSuccess) return cuda_fail(e, "short conv launch");
    if (state_out) {
        const dim3 g2((C + kConvThreads - 1) / kConvThreads, B);
        e = launch_pdl(short_conv_state_kernel<W>, g2, dim3(kConvThreads), 0, st, x, ld_x, T, C, state_in, state_out);
        if (e != cudaSuccess) return cuda_fail(e, "short conv state launch");
    }
    return NVFP4_OK;
}

}  // namespace

nvfp4_status short_conv_launch(const float* x, int64_t ld_x, int B, int64_t T, int C, int W, const float* w,
                               const float* state_in, float* state_out, float* out, int64_t ld_out, cudaStream_t st) {
    switch (W) {
        case 2: return launch_conv<2>(x, ld_x, B, T, C, w, state_in, state_out, out, ld_out, st);
        case 3: return launch_conv<3>(x, ld_x, B, T, C, w, state_in, state_out, out, ld_out, st);
        case 4: return launch_conv<4>(x, ld_x, B, T, C, w, state_in, state_out, out, ld_out, st);
        default: return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "conv width must be 2, 3 or 4");
    }
}

}  // namespace nvg

extern "C" nvfp4_status gdn_short_conv(const float* x, int64_t ld_x, int32_t B, int64_t T, int32_t C, int32_t W,
                                       const float* w, const float* state_in, float* state_out, float* out,
                                       int64_t ld_out, nvfp4_stream_t stream) {
    using namespace nvg;
    if (!x || !w || !out) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
    if (B < 1 || T < 1 || C < 1) return fail(NVFP4_ERR_INVALID_ARG, "B, T and C must be >= 1");
    if (W < 2 || W > 4) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "conv width must be 2, 3 or 4");
    if (ld_x < C || ld_out < C) return fail(NVFP4_ERR_INVALID_ARG, "ld_x / ld_out smaller than C");
    if (static_cast<int64_t>(B) * T > (int64_t(1) << 31) || (T + kConvTokens4 - 1) / kConvTokens4 > 65535 || B > 65535)
        return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "B or T too large");
    const char* xb = reinterpret_cast<const char*>(x);
    const char* ob = reinterpret_cast<const char*>(out);
    if (ob < xb + static_cast<int64_t>(B) * T * ld_x * 4 && xb < ob + static_cast<int64_t>(B) * T * ld_out * 4)
        return fail(NVFP4_ERR_INVALID_ARG, "out must not overlap x");
    return short_conv_launch(x, ld_x, B, T, C, W, w, state_in, state_out, out, ld_out, as_stream(stream));
}
