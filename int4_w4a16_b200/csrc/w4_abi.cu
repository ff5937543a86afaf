// w4_abi.cu -- host-side pieces of the C ABI shared by all entry points:
// version, status strings, CUDA error bookkeeping, the device status word and
// tensor-map encoding through the runtime's driver entry point.
#include <mutex>

#include "w4_common.cuh"

namespace w4host {

static thread_local int t_last_cuda_error = 0;

void set_cuda_error(cudaError_t e) { t_last_cuda_error = (int)e; }

int num_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    static int cached[64] = {0};
    if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev >= 0 && dev < 64) cached[dev] = n;
    return n;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

CUresult encode_tiled(CUtensorMap *map, CUtensorMapDataType dtype, cuuint32_t rank, void *gaddr,
                      const cuuint64_t *dims, const cuuint64_t *strides_bytes,
                      const cuuint32_t *box, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return CUDA_ERROR_NOT_FOUND;
    cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
    return fn(map, dtype, rank, gaddr, dims, strides_bytes, box, elem_strides,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace w4host

extern "C" int w4_version(void) { return 100; }

extern "C" const char *w4_status_string(w4_status s) {
    switch (s) {
        case W4_OK: return "W4_OK";
        case W4_ERR_INVALID_ARG: return "W4_ERR_INVALID_ARG";
        case W4_ERR_UNSUPPORTED: return "W4_ERR_UNSUPPORTED";
        case W4_ERR_CUDA: return "W4_ERR_CUDA";
        case W4_ERR_TIMEOUT: return "W4_ERR_TIMEOUT";
    }
    return "W4_ERR_UNKNOWN";
}

extern "C" int w4_last_cuda_error(void) { return w4host::t_last_cuda_error; }

extern "C" w4_status w4_device_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) {
        w4host::set_cuda_error(e);
        return W4_ERR_CUDA;
    }
    unsigned int flag = 0, flag_gemv = 0;
    e = w4host::gemm_device_status(&flag);
    if (e == cudaSuccess) e = w4host::gemv_device_status(&flag_gemv);
    flag |= flag_gemv;
    if (e != cudaSuccess) {
        w4host::set_cuda_error(e);
        return W4_ERR_CUDA;
    }
    return (flag & w4::kStatusTimeout) ? W4_ERR_TIMEOUT : W4_OK;
}
