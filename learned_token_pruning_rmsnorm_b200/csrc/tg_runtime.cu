// Host-side runtime pieces shared by the kernels: TMA descriptor encoding and
// the device status word.

#include <cuda.h>

#include <mutex>

#include "tg_sm100.cuh"

namespace tg {
namespace {

// One status word per device that loads the library.  Kernels OR error bits
// into it; tg_device_status reads and clears it.
__device__ int g_status_word;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
std::mutex g_status_mu;

}  // namespace

bool encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                         uint32_t box_inner, uint32_t box_outer) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int* device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_status_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    return g_status_ptr[dev];
}

namespace {

// One CTA whose waiting thread blocks on an mbarrier that nothing ever
// completes: the bounded wait must give up after timeout_ns, raise the abort
// flag and record TG_DEVICE_TIMEOUT, and the kernel must then return.
__global__ void selftest_wait_kernel(uint64_t timeout_ns, int* status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(sm100::smem_u32(&bar), 1);
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        sm100::mbar_wait(sm100::smem_u32(&bar), 0, &abort_flag, status, TG_WHERE_SOFTMAX, timeout_ns);
    __syncthreads();
}

}  // namespace

cudaError_t launch_selftest_wait(int64_t timeout_ns, cudaStream_t st) {
    int* status = device_status_ptr();
    if (!status) return cudaErrorInvalidSymbol;
    selftest_wait_kernel<<<1, 32, 0, st>>>(static_cast<uint64_t>(timeout_ns), status);
    return cudaGetLastError();
}

cudaError_t read_device_status(int32_t* word, bool clear, cudaStream_t st) {
    int* status = device_status_ptr();
    if (!status) return cudaErrorInvalidSymbol;
    cudaError_t e = cudaMemcpyAsync(word, status, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && clear) {
        e = cudaMemsetAsync(status, 0, sizeof(int32_t), st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    return e;
}

}  // namespace tg
