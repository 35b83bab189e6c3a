// Host-side helpers and the status / version entry points of libzb.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <mutex>

#include "zb_host.h"

namespace zb {

// One status word per device (each device holds its own copy of this symbol).
__device__ int g_status_word = 0;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceCache {
    bool ready = false;
    int sm_count = 0;
    int* status = nullptr;
};

std::mutex g_mu;
DeviceCache g_cache[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

}  // namespace

zb_status current_device(DeviceInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ZB_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ZB_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceCache& c = g_cache[dev];
    if (!c.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return ZB_ERR_CUDA;
        if (major != 10 || minor != 0) return ZB_ERR_DEVICE;
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess) return ZB_ERR_CUDA;
        c.sm_count = sms;
        c.status = static_cast<int*>(addr);
        c.ready = true;
    }
    out->device = dev;
    out->sm_count = c.sm_count;
    out->status = c.status;
    return ZB_OK;
}

unsigned long long wait_timeout_ns() {
    static unsigned long long v = [] {
        const char* e = getenv("ZB_WAIT_TIMEOUT_NS");
        unsigned long long t = 2000000000ull;  // 2 s
        if (e && *e) {
            unsigned long long u = strtoull(e, nullptr, 10);
            if (u > 0) t = u;
        }
        return t;
    }();
    return v;
}

zb_status make_map_bf16_3d(CUtensorMap* map, const void* base, int inner, long long rows,
                           int outer, int box_rows) {
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                return ZB_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
    }
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                                static_cast<cuuint64_t>(outer)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * 2,
                                   static_cast<cuuint64_t>(inner) * 2 * static_cast<cuuint64_t>(rows)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(inner), static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ZB_OK : ZB_ERR_CUDA;
}

}  // namespace zb

using namespace zb;

extern "C" int32_t zb_abi_version(void) { return 101; }

extern "C" const char* zb_status_string(int32_t status) {
    switch (status) {
        case ZB_OK: return "ZB_OK";
        case ZB_ERR_NULL: return "ZB_ERR_NULL: a required pointer is NULL";
        case ZB_ERR_SHAPE: return "ZB_ERR_SHAPE: a size or count is out of range";
        case ZB_ERR_ALIGN: return "ZB_ERR_ALIGN: a pointer is not 16-byte aligned";
        case ZB_ERR_UNSUPPORTED: return "ZB_ERR_UNSUPPORTED: unsupported head_dim, tile or size";
        case ZB_ERR_WORKSPACE: return "ZB_ERR_WORKSPACE: workspace missing or too small";
        case ZB_ERR_CUDA: return "ZB_ERR_CUDA: a CUDA call or kernel launch failed";
        case ZB_ERR_TIMEOUT: return "ZB_ERR_TIMEOUT: a bounded device-side wait gave up";
        case ZB_ERR_DEVICE: return "ZB_ERR_DEVICE: the current device is not an sm_100 GPU";
        case ZB_ERR_INDEX: return "ZB_ERR_INDEX: an index list was out of range or not ascending";
        case ZB_ERR_SINGULAR: return "ZB_ERR_SINGULAR: a least-squares system was not positive definite";
        default: return "unknown zb_status";
    }
}

extern "C" zb_status zb_last_device_status(void* stream) {
    DeviceInfo dev;
    zb_status e = current_device(&dev);
    if (e != ZB_OK) return e;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ZB_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, dev.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return ZB_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpy(dev.status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
            return ZB_ERR_CUDA;
    }
    return static_cast<zb_status>(word);
}
