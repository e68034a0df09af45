// quantize.cu -- online NVFP4 quantisation (E2M1 codes, E4M3 per-16 block
// scales in the tensor-core atom layout, FP32 per-tensor scale from amax).
//
// Format: review page of "Why Gated DeltaNet Survives 4-Bit Quantization",
// background section (paper sec.1): E2M1 values, one E4M3 scale per 16
// elements, one FP32 scale per tensor; the per-tensor scale is derived from the
// tensor itself at run time (the SoloQ summary page's dynamic NVFP4 variant).
//
// Two launches: (1) a grid-wide amax (128-bit loads, warp max, one atomicMax
// per CTA); (2) a grid-stride walk over the 512-byte scale atoms (128 rows x 64
// columns), one thread per four 16-element blocks, the scale bytes of an atom
// stored as four coalesced 128-byte rows.
#include <cuda_bf16.h>

#include "common.cuh"

namespace nvg {

namespace {

constexpr float kTwoPowMinus100 = 7.8886090522101181e-31f;  // 2^-100

// Decode an E4M3 byte (sign 0) to float, exactly.
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    if (e == 0) return static_cast<float>(m) * 0.001953125f;  // m * 2^-9, exact
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// fp32 -> E4M3, round to nearest even, saturating at 448 (non-negative input).
__device__ __forceinline__ uint32_t f32_to_e4m3(float s) {
    uint16_t r;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\t"
        "mov.b16 %0, t;\n\t}\n"
        : "=h"(r)
        : "f"(0.0f), "f"(s));
    return static_cast<uint32_t>(r) & 0xFFu;
}

// Eight fp32 values -> eight E2M1 codes packed in 32 bits, element 0 in the
// lowest nibble; round to nearest even, saturating at +-6.
__device__ __forceinline__ uint32_t f32x8_to_e2m1(const float (&y)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}\n"
        : "=r"(r)
        : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
    return r;
}

__device__ __forceinline__ float global_scale_from_amax(float amax) {
    return (amax < kTwoPowMinus100) ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int kPer16B = 8;
};
template <>
struct Vec<float> {
    static constexpr int kPer16B = 4;
};

__device__ __forceinline__ void unpack16B(const uint4& u, float* out, const __nv_bfloat16*) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        out[2 * i] = __uint_as_float(w[i] << 16);
        out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ void unpack16B(const uint4& u, float* out, const float*) {
    out[0] = __uint_as_float(u.x);
    out[1] = __uint_as_float(u.y);
    out[2] = __uint_as_float(u.z);
    out[3] = __uint_as_float(u.w);
}

// Pass 1: amax over the matrix into *amax_bits (float bits of a non-negative
// value, so unsigned order is float order).  Each warp walks whole rows, its lanes
// striding along the row with eight 16-byte loads in flight; warp max, then one
// atomicMax per CTA.
template <typename T>
__global__ void __launch_bounds__(256) amax_kernel(const T* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                                                   unsigned int* __restrict__ amax_bits) {
    constexpr int P = Vec<T>::kPer16B;
    constexpr int U = 8;
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t nvec = cols / P;   // 16-byte vectors per row
    float m = 0.0f;
    for (int64_t r = warp0; r < rows; r += nwarps) {
        const uint4* row = reinterpret_cast<const uint4*>(x + r * ld);
        int64_t c = lane;
        for (; c + 32 * (U - 1) < nvec; c += 32 * U) {
            uint4 u[U];
#pragma unroll
            for (int j = 0; j < U; ++j) u[j] = __ldg(row + c + 32 * j);
#pragma unroll
            for (int j = 0; j < U; ++j) {
                float f[8];
                unpack16B(u[j], f, x);
#pragma unroll
                for (int e = 0; e < P; ++e) m = fmaxf(m, fabsf(f[e]));
            }
        }
        for (; c < nvec; c += 32) {
            float f[8];
            unpack16B(__ldg(row + c), f, x);
#pragma unroll
            for (int e = 0; e < P; ++e) m = fmaxf(m, fabsf(f[e]));
        }
    }
    unsigned int b = __float_as_uint(m);
    b = __reduce_max_sync(0xffffffffu, b);
    __shared__ unsigned int warp_max[8];
    if (lane == 0) warp_max[threadIdx.x >> 5] = b;
    __syncthreads();
    if (threadIdx.x < 32) {
        unsigned int v = threadIdx.x < (blockDim.x >> 5) ? warp_max[threadIdx.x] : 0u;
        v = __reduce_max_sync(0xffffffffu, v);
        if (threadIdx.x == 0) atomicMax(amax_bits, v);
    }
}

// Pass 2: CTAs of 128 threads walk the scale atoms (128 rows x 64 columns, 512
// blocks of 16) in a grid-stride loop.  Thread t owns atom bytes t, t+128, t+256,
// t+384, i.e. the blocks (r, j) with r % 32 = (byte >> 4), r / 32 = (byte >> 2) & 3,
// j = byte & 3; all four blocks' loads are issued before any is used, and each
// group of 128 scale bytes is one coalesced store.
constexpr int kQuantThreads = 128;
constexpr int kQuantBPT = 512 / kQuantThreads;

template <typename T>
__global__ void __launch_bounds__(kQuantThreads) quant_kernel(const T* __restrict__ x, int64_t rows, int64_t cols,
                                                              int64_t ld, const unsigned int* __restrict__ amax_bits,
                                                              float* __restrict__ global_scale, int given_scale,
                                                              uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
    constexpr int P = Vec<T>::kPer16B;
    constexpr int NV = 16 / P;   // 16-byte loads per block
    const int64_t k_atoms = cols / 64;
    const int64_t natoms = ((rows + 127) / 128) * k_atoms;
    const int t = threadIdx.x;

    float S;
    if (given_scale) {
        S = *global_scale;
    } else {
        S = global_scale_from_amax(__uint_as_float(*amax_bits));
        if (blockIdx.x == 0 && t == 0) *global_scale = S;
    }
    const float d6 = __fmul_rn(6.0f, S);

    for (int64_t atom = blockIdx.x; atom < natoms; atom += gridDim.x) {
        const int64_t rb = atom / k_atoms, ka = atom - rb * k_atoms;
        uint4 u[kQuantBPT][NV];
        int64_t r[kQuantBPT], kb[kQuantBPT];
#pragma unroll
        for (int i = 0; i < kQuantBPT; ++i) {
            const int byte = t + i * kQuantThreads;
            r[i] = rb * 128 + (byte >> 4) + 32 * ((byte >> 2) & 3);
            kb[i] = ka * 4 + (byte & 3);
            const uint4* src = reinterpret_cast<const uint4*>(x + (r[i] < rows ? r[i] : 0) * ld + kb[i] * 16);
#pragma unroll
            for (int j = 0; j < NV; ++j) u[i][j] = r[i] < rows ? __ldg(src + j) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < kQuantBPT; ++i) {
            float v[16];
#pragma unroll
            for (int j = 0; j < NV; ++j) unpack16B(u[i][j], v + j * P, x);
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) m = fmaxf(m, fabsf(v[j]));
            const uint32_t sb = f32_to_e4m3(__fdiv_rn(m, d6));
            const float dec = __fmul_rn(e4m3_to_f32(sb), S);
            uint2 packed = make_uint2(0u, 0u);
            if (dec != 0.0f) {
                const float inv = __frcp_rn(dec);
                float y0[8], y1[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    y0[j] = __fmul_rn(v[j], inv);
                    y1[j] = __fmul_rn(v[8 + j], inv);
                }
                packed.x = f32x8_to_e2m1(y0);
                packed.y = f32x8_to_e2m1(y1);
            }
            if (r[i] < rows) *reinterpret_cast<uint2*>(codes + r[i] * (cols / 2) + kb[i] * 8) = packed;
            sf[atom * 512 + t + i * kQuantThreads] = static_cast<uint8_t>(r[i] < rows ? sb : 0u);
        }
    }
}

}  // namespace

nvfp4_status quantize_launch(const void* x, int32_t x_dtype, int64_t rows, int64_t cols, int64_t ld,
                             const nvfp4_tensor& out, int32_t flags, void* workspace, cudaStream_t st) {
    const bool given = flags == NVFP4_QUANT_GIVEN_SCALE;
    unsigned int* amax = static_cast<unsigned int*>(workspace);
    if (!given && flags != kQuantFromAmax) {
        cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned int), st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(amax)");
        // one warp per row, up to 8 resident CTAs of 8 warps per SM
        int64_t blocks = (rows + 7) / 8;
        const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
        if (blocks > cap) blocks = cap;
        if (x_dtype == NVFP4_DTYPE_BF16)
            amax_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), rows,
                                                                          cols, ld, amax);
        else
            amax_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(static_cast<const float*>(x), rows, cols, ld, amax);
    }
    const int64_t atoms = ((rows + 127) / 128) * (cols / 64);
    int64_t qblocks = static_cast<int64_t>(num_sms()) * 12;
    if (qblocks > atoms) qblocks = atoms;
    if (x_dtype == NVFP4_DTYPE_BF16)
        quant_kernel<__nv_bfloat16><<<(unsigned)qblocks, kQuantThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(x), rows, cols,
                                                                      ld, amax, out.global_scale, given ? 1 : 0,
                                                                      out.codes, out.sf);
    else
        quant_kernel<float><<<(unsigned)qblocks, kQuantThreads, 0, st>>>(static_cast<const float*>(x), rows, cols, ld, amax,
                                                              out.global_scale, given ? 1 : 0, out.codes, out.sf);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
    return NVFP4_OK;
}

nvfp4_status validate_tensor(const nvfp4_tensor* t, const char* name) {
    if (!t) return fail(NVFP4_ERR_INVALID_ARG, std::string(name) + " is null");
    if (!t->codes || !t->sf || !t->global_scale)
        return fail(NVFP4_ERR_INVALID_ARG, std::string(name) + " has a null buffer");
    if (t->rows < 1 || t->cols < 64) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, std::string(name) + " shape too small");
    if (t->cols % 64) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, std::string(name) + " cols must be a multiple of 64");
    if (t->rows > (int64_t(1) << 31) - 256 || t->cols > (int64_t(1) << 24))
        return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, std::string(name) + " too large");
    if (!aligned16(t->codes) || !aligned16(t->sf))
        return fail(NVFP4_ERR_MISALIGNED, std::string(name) + " buffers must be 16-byte aligned");
    return NVFP4_OK;
}

}  // namespace nvg

extern "C" size_t nvfp4_sf_bytes(int64_t rows, int64_t cols) {
    if (rows < 1 || cols < 16) return 0;
    return static_cast<size_t>((rows + 127) / 128 * 128) * static_cast<size_t>(cols / 16);
}

extern "C" size_t nvfp4_quantize_workspace_size(void) { return 256; }

extern "C" nvfp4_status nvfp4_quantize(const void* x, int32_t x_dtype, int64_t rows, int64_t cols, int64_t ld,
                                       const nvfp4_tensor* out, int32_t flags, void* workspace,
                                       size_t workspace_bytes, nvfp4_stream_t stream) {
    using namespace nvg;
    if (!x) return fail(NVFP4_ERR_INVALID_ARG, "x is null");
    if (x_dtype != NVFP4_DTYPE_BF16 && x_dtype != NVFP4_DTYPE_FP32) return fail(NVFP4_ERR_INVALID_ARG, "bad x_dtype");
    if (flags != NVFP4_QUANT_COMPUTE_SCALE && flags != NVFP4_QUANT_GIVEN_SCALE)
        return fail(NVFP4_ERR_INVALID_ARG, "bad flags");
    nvfp4_status s = validate_tensor(out, "out");
    if (s != NVFP4_OK) return s;
    if (out->rows != rows || out->cols != cols) return fail(NVFP4_ERR_INVALID_ARG, "out shape differs from x");
    if (ld < cols) return fail(NVFP4_ERR_INVALID_ARG, "ld < cols");
    const int64_t esz = x_dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
    if (!aligned16(x) || (ld * esz) % 16) return fail(NVFP4_ERR_MISALIGNED, "x / ld not 16-byte aligned");
    if (flags == NVFP4_QUANT_COMPUTE_SCALE &&
        (!workspace || workspace_bytes < nvfp4_quantize_workspace_size() || !aligned16(workspace)))
        return fail(NVFP4_ERR_WORKSPACE, "quantize workspace missing or too small");
    return quantize_launch(x, x_dtype, rows, cols, ld, *out, flags, workspace, as_stream(stream));
}
