// scan_noalloc.cu -- gdn_scan_noalloc: the chunked delta-rule scan with its
// scratch in a fixed device array owned by this library, for callers that
// cannot allocate device memory themselves (for example a plugin running
// inside a host framework that owns every allocation, or code that must not
// call cudaMalloc while a stream is being captured into a CUDA graph).
//
// The chunked scan needs per-(sequence, head, 64-token chunk) scratch (W~, U~,
// the masked decayed Q K^T and the running log-decay).  Here that scratch is
// the file-scope array below: kNoAllocScratchBytes on every GPU that loads the
// library, held until the process exits.  Problems whose scratch would not fit
// are rejected before anything is launched.
#include <mutex>

#include "common.cuh"

namespace nvg {

size_t scan_workspace_bytes(int B, int64_t T, const gdn_dims& d, int algo);
nvfp4_status validate_dims(const gdn_dims* d);
nvfp4_status scan_launch(const float* q, const float* k, const float* v, int64_t ld_v, const float* g,
                         const float* beta, int B, int64_t T, const gdn_dims& d, float scale, int form, int algo,
                         const float* s_in, float* s_out, float* o, void* ws, cudaStream_t st,
                         unsigned int* o_amax, int64_t ld_qk, int normalize_qk);

namespace {

constexpr size_t kNoAllocScratchBytes = GDN_SCAN_NOALLOC_MAX_SCRATCH_BYTES;

// Host code must not pass this symbol to a kernel: on the host it names a
// stand-in object, not device memory.  Its device address is looked up below.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached.
nvfp4_status scratch_address(void** out) {
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(NVFP4_ERR_CUDA, "device ordinal out of range");
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(noalloc scratch)");
        addr[dev] = p;
    }
    *out = addr[dev];
    return NVFP4_OK;
}

}  // namespace

}  // namespace nvg

extern "C" nvfp4_status gdn_scan_noalloc(const float* q_hat, const float* k_hat, const float* v, int64_t ld_v,
                                         const float* g, const float* beta, int32_t B, int64_t T,
                                         const gdn_dims* dims, float scale, int32_t form, const float* state_in,
                                         float* state_out, float* o, nvfp4_stream_t stream) {
    using namespace nvg;
    nvfp4_status s = validate_dims(dims);
    if (s != NVFP4_OK) return s;
    if (!q_hat || !k_hat || !v || !g || !beta || !o) return fail(NVFP4_ERR_INVALID_ARG, "null pointer");
    if (B < 1 || T < 1) return fail(NVFP4_ERR_INVALID_ARG, "B and T must be >= 1");
    if (form != GDN_FORM_PAGES && form != GDN_FORM_STANDARD) return fail(NVFP4_ERR_INVALID_ARG, "bad form");
    if (ld_v < static_cast<int64_t>(dims->Hv) * dims->V) return fail(NVFP4_ERR_INVALID_ARG, "ld_v < Hv*V");
    if (static_cast<int64_t>(B) * T > (int64_t(1) << 31)) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "B*T too large");
    if (!aligned16(q_hat) || !aligned16(k_hat) || !aligned16(o) || !aligned16(v) || ld_v % 4)
        return fail(NVFP4_ERR_MISALIGNED, "q_hat, k_hat, v, o must be 16-byte aligned and ld_v % 4 == 0");
    if (!aligned16(state_in) || !aligned16(state_out))   // the chunked kernel moves the state as float4
        return fail(NVFP4_ERR_MISALIGNED, "state_in and state_out must be 16-byte aligned");
    const size_t need = scan_workspace_bytes(B, T, *dims, GDN_SCAN_CHUNKED);
    if (need > kNoAllocScratchBytes)
        return fail(NVFP4_ERR_WORKSPACE, "gdn_scan_noalloc: this problem needs " + std::to_string(need) +
                                             " bytes of scratch, more than the library's fixed " +
                                             std::to_string(kNoAllocScratchBytes) +
                                             "-byte array; use gdn_scan with a caller-provided workspace");
    void* scratch = nullptr;
    if ((s = scratch_address(&scratch)) != NVFP4_OK) return s;
    return scan_launch(q_hat, k_hat, v, ld_v, g, beta, B, T, *dims, scale, form, GDN_SCAN_CHUNKED, state_in,
                       state_out, o, scratch, as_stream(stream), nullptr, static_cast<int64_t>(dims->Hk) * dims->K,
                       0);
}
