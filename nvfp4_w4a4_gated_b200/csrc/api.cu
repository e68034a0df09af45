// api.cu -- status plumbing, device error word, TMA descriptor encoding.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>
#include <string>

#include "common.cuh"

namespace nvg {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

nvfp4_status fail(nvfp4_status st, const std::string& msg) {
    g_last_error = msg;
    return st;
}

nvfp4_status cuda_fail(cudaError_t e, const char* what) {
    g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
    return NVFP4_ERR_CUDA;
}

// One word per device: kernels OR failure codes into it.
__device__ unsigned int g_device_error_word;

unsigned int* device_error_word() {
    static std::mutex mu;
    static unsigned int* ptrs[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<unsigned int*>(p);
    }
    return ptrs[dev];
}

int num_sms() {
    // per device; threads may race to fill a slot, and all store the same value
    static std::atomic<int> cached[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    int v = cached[dev].load(std::memory_order_relaxed);
    if (!v) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        v = n > 0 ? n : 148;
        cached[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

nvfp4_status make_tmap_u8_sw128(CUtensorMap* map, const void* base, uint64_t rows, uint64_t row_bytes,
                                uint32_t box_rows, uint32_t box_bytes) {
    auto fn = encode_fn();
    if (!fn) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {row_bytes, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_bytes, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string(r));
    return NVFP4_OK;
}

nvfp4_status make_tmap_f32_sw128(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                                 uint32_t box_rows, uint32_t box_cols) {
    auto fn = encode_fn();
    if (!fn) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 4};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled(f32) failed: " + std::to_string(r));
    return NVFP4_OK;
}

}  // namespace nvg

extern "C" const char* nvfp4_last_error(void) { return nvg::g_last_error.c_str(); }

namespace nvg {
namespace {
// One thread waits, bounded, on an mbarrier no one arrives on (see the header).
__global__ void selftest_wait_kernel(uint32_t budget_cycles, unsigned int* err) {
    __shared__ uint64_t bar;
    mbar_init(&bar, 1);
    fence_mbar_init();
    const long long t0 = clock64();
    while (!mbar_try_wait(&bar, 0)) {
        if (clock64() - t0 > static_cast<long long>(budget_cycles)) {
            atomicOr(err, kErrTimeoutSelftest);
            return;
        }
    }
}
}  // namespace
}  // namespace nvg

extern "C" nvfp4_status nvfp4_selftest_wait_timeout(uint32_t budget_cycles, nvfp4_stream_t stream) {
    using namespace nvg;
    if (budget_cycles < 1 || budget_cycles > (1u << 30)) return fail(NVFP4_ERR_INVALID_ARG, "budget_cycles out of range");
    unsigned int* err = device_error_word();
    if (!err) return fail(NVFP4_ERR_CUDA, "device error word unavailable");
    selftest_wait_kernel<<<1, 1, 0, as_stream(stream)>>>(budget_cycles, err);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
    return NVFP4_OK;
}

extern "C" const char* nvfp4_version(void) { return "0.1.0"; }

extern "C" nvfp4_status nvfp4_check_device_error(nvfp4_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(nvg::as_stream(stream));
    if (e != cudaSuccess) return nvg::cuda_fail(e, "cudaStreamSynchronize");
    unsigned int* w = nvg::device_error_word();
    if (!w) return nvg::fail(NVFP4_ERR_CUDA, "device error word unavailable");
    unsigned int v = 0;
    e = cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return nvg::cuda_fail(e, "read device error word");
    if (v != 0) {
        unsigned int z = 0;
        cudaMemcpy(w, &z, sizeof(z), cudaMemcpyHostToDevice);
        return nvg::fail(NVFP4_ERR_TIMEOUT, "a kernel's bounded wait ran out (code " + std::to_string(v) + ")");
    }
    return NVFP4_OK;
}
