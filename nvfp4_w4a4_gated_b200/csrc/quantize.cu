// quantize.cu -- online NVFP4 quantisation (E2M1 codes, E4M3 per-16 block
// scales in the tensor-core atom layout, FP32 per-tensor scale from amax).
//
// Format: review page of "Why Gated DeltaNet Survives 4-Bit Quantization",
// background section (paper sec.1): E2M1 values, one E4M3 scale per 16
// elements, one FP32 scale per tensor; the per-tensor scale is derived from the
// tensor itself at run time (the SoloQ summary page's dynamic NVFP4 variant).
//
// One cooperative launch: an amax pass over the 512-byte scale atoms (128 rows
// x 64 columns), a grid barrier, then the quantisation pass over the same atoms
// in reverse order (their data still in L2), one thread per four 16-element
// blocks, the scale bytes of an atom stored as four coalesced 128-byte rows.
// If the grid cannot be co-resident, a separate amax launch runs first.
#include <atomic>
#include <cuda_bf16.h>

#include <type_traits>

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
    pdl_wait_and_trigger();
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

// Zeroes n 32-bit words (the quantiser's amax and arrival words).  A kernel rather
// than a memset, so that it chains with its neighbours by programmatic launch.
__global__ void __launch_bounds__(32) zero_words_kernel(unsigned int* __restrict__ w, int n) {
    pdl_wait_and_trigger();
    if (static_cast<int>(threadIdx.x) < n) w[threadIdx.x] = 0u;
}

// Pass 2 (and, fused, pass 1): the matrix is cut into scale atoms (128 rows x
// 64 columns, 512 blocks of 16).  A group of 128 threads handles one atom at a
// time: thread t owns atom bytes t, t+128, t+256, t+384, i.e. the blocks (r, j)
// with r % 32 = (byte >> 4), r / 32 = (byte >> 2) & 3, j = byte & 3; all four
// blocks' loads are issued before any is used, and each group of 128 scale bytes
// is one coalesced store.  A CTA holds kQuantGroups such groups.
constexpr int kQuantGroupThreads = 128;
constexpr int kQuantBPT = 512 / kQuantGroupThreads;
constexpr int kQuantGroups = 2;
constexpr int kQuantThreads = kQuantGroupThreads * kQuantGroups;
constexpr unsigned int kQuantSpinLimit = 1u << 22;   // x ~100 ns per poll: ~0.4 s

template <typename T>
struct AtomRegs {
    static constexpr int NV = 16 / Vec<T>::kPer16B;   // 16-byte loads per block
    uint4 u[kQuantBPT][NV];
    int64_t r[kQuantBPT], kb[kQuantBPT];
};

template <typename T>
__device__ __forceinline__ void atom_load(const T* __restrict__ x, int64_t rows, int64_t ld, int64_t k_atoms,
                                          int64_t atom, int t, AtomRegs<T>& a) {
    const int64_t rb = atom / k_atoms, ka = atom - rb * k_atoms;
#pragma unroll
    for (int i = 0; i < kQuantBPT; ++i) {
        const int byte = t + i * kQuantGroupThreads;
        a.r[i] = rb * 128 + (byte >> 4) + 32 * ((byte >> 2) & 3);
        a.kb[i] = ka * 4 + (byte & 3);
        const uint4* src = reinterpret_cast<const uint4*>(x + (a.r[i] < rows ? a.r[i] : 0) * ld + a.kb[i] * 16);
#pragma unroll
        for (int j = 0; j < AtomRegs<T>::NV; ++j)
            a.u[i][j] = a.r[i] < rows ? __ldg(src + j) : make_uint4(0u, 0u, 0u, 0u);
    }
}

// Running |x| maximum over raw 16-byte vectors.  bf16: the magnitudes' bit
// patterns (sign cleared) order like the values, so two are compared at a time
// with one unsigned 16x2 max; the accumulator holds two 16-bit maxima.  fp32:
// one max with an absolute-value operand per element.
struct AbsMaxBf16 {
    uint32_t acc = 0;
    __device__ __forceinline__ void add(const uint4& u) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) asm("max.u16x2 %0, %0, %1;" : "+r"(acc) : "r"(w[i] & 0x7FFF7FFFu));
    }
    __device__ __forceinline__ float value() const {
        const uint32_t m = max(acc & 0xFFFFu, acc >> 16);
        return __uint_as_float(m << 16);
    }
};
struct AbsMaxF32 {
    float acc = 0.0f;
    __device__ __forceinline__ void add(const uint4& u) {
        acc = fmaxf(acc, fabsf(__uint_as_float(u.x)));
        acc = fmaxf(acc, fabsf(__uint_as_float(u.y)));
        acc = fmaxf(acc, fabsf(__uint_as_float(u.z)));
        acc = fmaxf(acc, fabsf(__uint_as_float(u.w)));
    }
    __device__ __forceinline__ float value() const { return acc; }
};
template <typename T>
struct AbsMaxOf;
template <>
struct AbsMaxOf<__nv_bfloat16> {
    using type = AbsMaxBf16;
};
template <>
struct AbsMaxOf<float> {
    using type = AbsMaxF32;
};

template <typename T>
__device__ __forceinline__ void atom_absmax(const AtomRegs<T>& a, typename AbsMaxOf<T>::type& m) {
#pragma unroll
    for (int i = 0; i < kQuantBPT; ++i)
#pragma unroll
        for (int j = 0; j < AtomRegs<T>::NV; ++j) m.add(a.u[i][j]);
}

// Two fp32 products x * s, each rounded to nearest even (one packed multiply),
// then the pair's E2M1 codes as one byte, element x0 in the low nibble.
__device__ __forceinline__ uint32_t scale_pair_to_e2m1(float x0, float x1, float s) {
    uint16_t r;
    asm("{\n\t.reg .b64 xv, sv, yv;\n\t.reg .f32 y0, y1;\n\t.reg .b8 c;\n\t"
        "mov.b64 xv, {%1, %2};\n\t"
        "mov.b64 sv, {%3, %3};\n\t"
        "mul.rn.f32x2 yv, xv, sv;\n\t"
        "mov.b64 {y0, y1}, yv;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c, y1, y0;\n\t"
        "cvt.u16.u8 %0, c;\n\t}\n"
        : "=h"(r)
        : "f"(x0), "f"(x1), "f"(s));
    return r;
}

// One 16-element block from its raw vectors: block scale byte and 8 code bytes.
__device__ __forceinline__ uint2 block_codes(const uint4 (&u)[2], float inv, const __nv_bfloat16*) {
    const uint32_t w[8] = {u[0].x, u[0].y, u[0].z, u[0].w, u[1].x, u[1].y, u[1].z, u[1].w};
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        b[i] = scale_pair_to_e2m1(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u), inv);
    return make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24), b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
}
__device__ __forceinline__ uint2 block_codes(const uint4 (&u)[4], float inv, const float*) {
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        b[2 * i] = scale_pair_to_e2m1(__uint_as_float(u[i].x), __uint_as_float(u[i].y), inv);
        b[2 * i + 1] = scale_pair_to_e2m1(__uint_as_float(u[i].z), __uint_as_float(u[i].w), inv);
    }
    return make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24), b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
}

// Block scale of a block with |x| maximum m: the E4M3 rounding (nearest even,
// saturating) of the fp32 quotient RN(m / d6).  The quotient is formed without a
// divide: q0 = RN(m * y) with y = RN(1 / d6), then one Newton-Markstein
// correction q1 = RN(q0 + r * y) with the exact remainder r = m - q0 * d6 (one
// fma).  q1 is within an ulp of the true quotient, so its E4M3 rounding can
// differ from that of RN(m / d6) only where the quotient lies within an ulp of
// an E4M3 rounding midpoint.  Every midpoint (and every E4M3 value) has at most
// five significant bits, i.e. its low 19 mantissa bits are zero; q1 within two
// ulps of such a number takes the correctly rounded division instead.
__device__ __forceinline__ uint32_t block_scale_byte(float m, float d6, float y6) {
    float q = __fmul_rn(m, y6);
    const float r = __fmaf_rn(-q, d6, m);
    q = __fmaf_rn(r, y6, q);
    if (((__float_as_uint(q) + 2u) & 0x7FFFFu) <= 4u) q = __fdiv_rn(m, d6);
    return f32_to_e4m3(q);
}

template <typename T>
__device__ __forceinline__ void atom_quantize_store(const AtomRegs<T>& a, int64_t rows, int64_t cols, int64_t atom,
                                                    int t, float d6, float y6, const float* __restrict__ s_inv,
                                                    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
#pragma unroll
    for (int i = 0; i < kQuantBPT; ++i) {
        typename AbsMaxOf<T>::type mx;
#pragma unroll
        for (int j = 0; j < AtomRegs<T>::NV; ++j) mx.add(a.u[i][j]);
        const uint32_t sb = block_scale_byte(mx.value(), d6, y6);
        const float inv = s_inv[sb & 0x7Fu];
        uint2 packed = make_uint2(0u, 0u);
        if (inv != 0.0f) packed = block_codes(a.u[i], inv, static_cast<const T*>(nullptr));
        if (a.r[i] < rows) *reinterpret_cast<uint2*>(codes + a.r[i] * (cols / 2) + a.kb[i] * 8) = packed;
        sf[atom * 512 + t + i * kQuantGroupThreads] = static_cast<uint8_t>(a.r[i] < rows ? sb : 0u);
    }
}

// Where the per-tensor scale comes from.
enum QuantScaleMode : int {
    kScaleFromAmaxWord = 0,   // S from the amax word a previous launch (or the scan) filled
    kScaleGiven = 1,          // S read from *global_scale
};

// kFindAmax: one launch does both passes.  Pass 1 takes the absmax of this
// group's atoms; after one atomicMax per CTA the CTAs meet at a grid barrier
// (an arrival counter, so the launch must be cooperative), and pass 2 then
// quantises the same atoms in reverse order, so the data read last in pass 1
// (still in L2) is read first; the very last atom of pass 1 stays in registers
// across the barrier and is quantised without a second read.  With bf16 input
// pass 2 loads the next atom before quantising the current one (two atoms in
// flight per thread); fp32 input has no registers to spare for that.
// ws[0] = amax bits, ws[1] = arrival counter, both zero at launch.  The barrier
// wait is bounded: on expiry the kernel sets kErrTimeoutQuant and carries on
// with whatever amax it sees.
template <typename T, bool kFindAmax>
__global__ void __launch_bounds__(kQuantThreads) quant_kernel(const T* __restrict__ x, int64_t rows, int64_t cols,
                                                              int64_t ld, unsigned int* __restrict__ ws,
                                                              float* __restrict__ global_scale, int scale_mode,
                                                              uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                              unsigned int* __restrict__ err) {
    pdl_wait_and_trigger();
    const int64_t k_atoms = cols / 64;
    const int64_t natoms = ((rows + 127) / 128) * k_atoms;
    const int t = threadIdx.x % kQuantGroupThreads;
    const int64_t group = static_cast<int64_t>(blockIdx.x) * kQuantGroups + threadIdx.x / kQuantGroupThreads;
    const int64_t ngroups = static_cast<int64_t>(gridDim.x) * kQuantGroups;
    __shared__ float s_scale;
    __shared__ unsigned int warp_max[kQuantThreads / 32];
    AtomRegs<T> cur;   // pass 1's last atom is pass 2's first

    if constexpr (kFindAmax) {
        typename AbsMaxOf<T>::type m;
        for (int64_t atom = group; atom < natoms; atom += ngroups) {
            atom_load(x, rows, ld, k_atoms, atom, t, cur);
            atom_absmax(cur, m);
        }
        const unsigned int b = __reduce_max_sync(0xffffffffu, __float_as_uint(m.value()));
        if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = b;
        __syncthreads();
        if (threadIdx.x < 32) {
            unsigned int v = threadIdx.x < kQuantThreads / 32 ? warp_max[threadIdx.x] : 0u;
            v = __reduce_max_sync(0xffffffffu, v);
            if (threadIdx.x == 0) {
                atomicMax(&ws[0], v);
                __threadfence();
                atomicAdd(&ws[1], 1u);
                unsigned int arrived = 0, polls = 0;
                for (;;) {
                    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(arrived) : "l"(ws + 1) : "memory");
                    if (arrived >= gridDim.x) break;
                    if (++polls > kQuantSpinLimit) {
                        atomicOr(err, kErrTimeoutQuant);
                        break;
                    }
                    __nanosleep(64);
                }
                unsigned int amax;
                asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(amax) : "l"(ws) : "memory");
                const float S = global_scale_from_amax(__uint_as_float(amax));
                s_scale = S;
                if (blockIdx.x == 0) *global_scale = S;
            }
        }
        __syncthreads();
    } else {
        if (threadIdx.x == 0) {
            const float S = scale_mode == kScaleGiven ? *global_scale : global_scale_from_amax(__uint_as_float(*ws));
            s_scale = S;
            if (blockIdx.x == 0 && scale_mode != kScaleGiven) *global_scale = S;
        }
        __syncthreads();
    }
    // The element multiplier of a block is RN(1 / RN(E4M3(sb) * S)); sb is one of
    // 127 finite non-negative E4M3 values (0x7F is NaN and never produced), so the
    // multipliers are tabulated once per CTA; 0 marks a block that decodes to 0.
    __shared__ float s_inv[128];
    const float S = s_scale;
    if (threadIdx.x < 128) {
        const float dec = __fmul_rn(e4m3_to_f32(threadIdx.x), S);
        s_inv[threadIdx.x] = dec != 0.0f ? __frcp_rn(dec) : 0.0f;
    }
    __syncthreads();
    const float d6 = __fmul_rn(6.0f, S);
    const float y6 = __frcp_rn(d6);
    if (group >= natoms) return;
    const int64_t last = group + ((natoms - 1 - group) / ngroups) * ngroups;
    const int64_t first = kFindAmax ? last : group, step = kFindAmax ? -ngroups : ngroups;
    auto in_range = [&](int64_t atom) { return kFindAmax ? atom >= group : atom < natoms; };
    if constexpr (!kFindAmax) atom_load(x, rows, ld, k_atoms, first, t, cur);
    constexpr bool kPrefetch = std::is_same<T, __nv_bfloat16>::value;
    for (int64_t atom = first; in_range(atom); atom += step) {
        if constexpr (kPrefetch) {
            AtomRegs<T> nxt;
            const bool more = in_range(atom + step);
            if (more) atom_load(x, rows, ld, k_atoms, atom + step, t, nxt);
            atom_quantize_store(cur, rows, cols, atom, t, d6, y6, s_inv, codes, sf);
            if (more) cur = nxt;
        } else {
            if (atom != first) atom_load(x, rows, ld, k_atoms, atom, t, cur);
            atom_quantize_store(cur, rows, cols, atom, t, d6, y6, s_inv, codes, sf);
        }
    }
}

template <typename T, bool kFindAmax>
int quant_blocks_per_sm() {
    // threads may race to fill it, and all store the same value
    static std::atomic<int> cached{0};
    int v = cached.load(std::memory_order_relaxed);
    if (!v) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, quant_kernel<T, kFindAmax>, kQuantThreads, 0) !=
                cudaSuccess ||
            n < 1)
            n = 1;
        v = n;
        cached.store(v, std::memory_order_relaxed);
    }
    return v;
}

template <typename T>
nvfp4_status quant_dispatch(const T* x, int64_t rows, int64_t cols, int64_t ld, const nvfp4_tensor& out,
                            int32_t flags, unsigned int* ws, cudaStream_t st) {
    unsigned int* err = device_error_word();
    if (!err) return fail(NVFP4_ERR_CUDA, "device error word unavailable");
    const int64_t atoms = ((rows + 127) / 128) * (cols / 64);
    const int64_t groups_needed = (atoms + kQuantGroups - 1) / kQuantGroups;
    cudaError_t e;
    if (flags == NVFP4_QUANT_AMAX_ONLY) {   // word 0 := max|x|, nothing else written
        e = launch_pdl(zero_words_kernel, dim3(1), dim3(32), 0, st, ws, 2);
        if (e != cudaSuccess) return cuda_fail(e, "zero amax words");
        int64_t blocks = (rows + 7) / 8;
        const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
        if (blocks > cap) blocks = cap;
        e = launch_pdl(amax_kernel<T>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, x, rows, cols, ld, ws);
        if (e != cudaSuccess) return cuda_fail(e, "amax launch");
        return NVFP4_OK;
    }
    if (flags == NVFP4_QUANT_COMPUTE_SCALE || flags == kQuantComputeZeroedWs) {
        if (flags == NVFP4_QUANT_COMPUTE_SCALE) {
            e = launch_pdl(zero_words_kernel, dim3(1), dim3(32), 0, st, ws, 2);
            if (e != cudaSuccess) return cuda_fail(e, "zero amax words");
        }
        // one launch: every CTA resident at once (cooperative launch), at most one
        // atom group per thread group
        int64_t grid = static_cast<int64_t>(num_sms()) * quant_blocks_per_sm<T, true>();
        if (grid > groups_needed) grid = groups_needed;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(kQuantThreads);
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, quant_kernel<T, true>, x, rows, cols, ld, ws, out.global_scale,
                               static_cast<int>(kScaleFromAmaxWord), out.codes, out.sf, err);
        if (e == cudaSuccess) return NVFP4_OK;
        if (e != cudaErrorCooperativeLaunchTooLarge && e != cudaErrorNotSupported)
            return cuda_fail(e, "quantize launch");
        (void)cudaGetLastError();
        // the device cannot hold the whole grid at once: two launches instead
        int64_t blocks = (rows + 7) / 8;
        const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
        if (blocks > cap) blocks = cap;
        e = launch_pdl(amax_kernel<T>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, x, rows, cols, ld, ws);
        if (e != cudaSuccess) return cuda_fail(e, "amax launch");
    }
    int64_t grid = static_cast<int64_t>(num_sms()) * quant_blocks_per_sm<T, false>();
    if (grid > groups_needed) grid = groups_needed;
    e = launch_pdl(quant_kernel<T, false>, dim3(static_cast<unsigned>(grid)), dim3(kQuantThreads), 0, st, x, rows,
                   cols, ld, ws, out.global_scale,
                   flags == NVFP4_QUANT_GIVEN_SCALE ? static_cast<int>(kScaleGiven)
                                                    : static_cast<int>(kScaleFromAmaxWord),
                   out.codes, out.sf, err);
    if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
    return NVFP4_OK;
}

}  // namespace

nvfp4_status zero_words_launch(unsigned int* w, int n, cudaStream_t st) {
    const cudaError_t e = launch_pdl(zero_words_kernel, dim3(1), dim3(32), 0, st, w, n);
    if (e != cudaSuccess) return cuda_fail(e, "zero words");
    return NVFP4_OK;
}

// flags: NVFP4_QUANT_COMPUTE_SCALE (amax and quantisation, one cooperative
// launch; kQuantComputeZeroedWs when the caller has zeroed workspace[0..1]),
// NVFP4_QUANT_AMAX_ONLY (workspace[0] := max|x| only),
// NVFP4_QUANT_GIVEN_SCALE (S read from out.global_scale), or
// kQuantFromAmax (S from the amax word at workspace[0], which a producer such
// as the scan has filled; the quantisation pass only).
nvfp4_status quantize_launch(const void* x, int32_t x_dtype, int64_t rows, int64_t cols, int64_t ld,
                             const nvfp4_tensor& out, int32_t flags, void* workspace, cudaStream_t st) {
    unsigned int* ws = static_cast<unsigned int*>(workspace);
    if (x_dtype == NVFP4_DTYPE_BF16)
        return quant_dispatch(static_cast<const __nv_bfloat16*>(x), rows, cols, ld, out, flags, ws, st);
    return quant_dispatch(static_cast<const float*>(x), rows, cols, ld, out, flags, ws, st);
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
    if (flags != NVFP4_QUANT_COMPUTE_SCALE && flags != NVFP4_QUANT_GIVEN_SCALE && flags != NVFP4_QUANT_AMAX_ONLY &&
        flags != NVFP4_QUANT_FROM_AMAX)
        return fail(NVFP4_ERR_INVALID_ARG, "bad flags");
    nvfp4_status s = validate_tensor(out, "out");
    if (s != NVFP4_OK) return s;
    if (out->rows != rows || out->cols != cols) return fail(NVFP4_ERR_INVALID_ARG, "out shape differs from x");
    if (ld < cols) return fail(NVFP4_ERR_INVALID_ARG, "ld < cols");
    const int64_t esz = x_dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
    if (!aligned16(x) || (ld * esz) % 16) return fail(NVFP4_ERR_MISALIGNED, "x / ld not 16-byte aligned");
    if (flags != NVFP4_QUANT_GIVEN_SCALE &&
        (!workspace || workspace_bytes < nvfp4_quantize_workspace_size() || !aligned16(workspace)))
        return fail(NVFP4_ERR_WORKSPACE, "quantize workspace missing or too small");
    return quantize_launch(x, x_dtype, rows, cols, ld, *out, flags == NVFP4_QUANT_FROM_AMAX ? kQuantFromAmax : flags,
                           workspace, as_stream(stream));
}
