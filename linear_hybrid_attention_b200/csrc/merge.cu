// Dense softmax attention with the keys split into equal parts, for query sets
// too small to fill the GPU (the calibration rows of the affine fit: 32 query
// tiles per head).  The dense kernel runs once over heads x splits "virtual
// heads" -- virtual head h * S + p sees keys [p N / S, (p + 1) N / S) of head
// h, which in the [H][N][d] layout is the same memory viewed as
// [H S][N / S][d] -- and writes fp32 partial outputs with their log-sum-exp;
// a merge kernel then forms each row's softmax over all N keys:
//   O = sum_p e^(lse_p - M) O_p / sum_p e^(lse_p - M),   lse = M + ln sum_p e^(lse_p - M),
// M = max_p lse_p (the partial softmaxes reweighted by their share of the
// total mass).  "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D
// Reconstruction", Abstract: the affine fit is closed-form against the dense
// layer's outputs on calibration rows.
#include <cuda_runtime.h>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace mrg {

constexpr int HD = 64;
constexpr int THREADS = 256;
constexpr int MAX_SPLITS = 16;

inline size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Layout {
    size_t qrep, op, lsep, total;
};
inline Layout layout(long long n_q, int heads, int splits) {
    const size_t rows = static_cast<size_t>(n_q) * heads * splits;
    Layout l;
    l.qrep = 0;
    l.op = al256(rows * HD * 2);
    l.lsep = l.op + al256(rows * HD * sizeof(float));
    l.total = l.lsep + al256(rows * sizeof(float));
    return l;
}

// One warp per (head, query row); lane l owns columns 2l and 2l + 1.
__global__ void __launch_bounds__(THREADS)
merge_kernel(const float* __restrict__ Op, const float* __restrict__ lsep, int heads, int splits, long long n_q,
             void* __restrict__ O, int out_fp32, float* __restrict__ lse) {
    const long long gw = static_cast<long long>(blockIdx.x) * (THREADS / 32) + (threadIdx.x >> 5);
    if (gw >= static_cast<long long>(heads) * n_q) return;
    const int lane = threadIdx.x & 31;
    const long long h = gw / n_q, r = gw % n_q;
    float M = -INFINITY;
    for (int p = 0; p < splits; ++p) M = fmaxf(M, lsep[(h * splits + p) * n_q + r]);
    float den = 0.f, o0 = 0.f, o1 = 0.f;
    for (int p = 0; p < splits; ++p) {
        const long long vr = (h * splits + p) * n_q + r;
        const float wgt = expf(lsep[vr] - M);
        const float2 v = reinterpret_cast<const float2*>(Op + vr * HD)[lane];
        den += wgt;
        o0 = fmaf(wgt, v.x, o0);
        o1 = fmaf(wgt, v.y, o1);
    }
    const float inv = 1.f / den;
    const long long orow = h * n_q + r;
    if (out_fp32) {
        reinterpret_cast<float2*>(static_cast<float*>(O) + orow * HD)[lane] = make_float2(o0 * inv, o1 * inv);
    } else {
        reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(O) + orow * HD)[lane] = pack_bf16x2(o0 * inv, o1 * inv);
    }
    if (lse && lane == 0) lse[orow] = M + logf(den);
}

}  // namespace mrg
}  // namespace zb

using namespace zb;

extern "C" size_t zb_dense_attn_split_workspace_bytes(int64_t n_q, int32_t heads, int32_t head_dim, int32_t splits) {
    if (n_q < 1 || heads < 1 || head_dim != mrg::HD || splits < 1 || splits > mrg::MAX_SPLITS) return 0;
    if (splits == 1) return 0;
    return mrg::layout(n_q, heads, splits).total;
}

extern "C" zb_status zb_dense_attn_split(const uint16_t* Q, int64_t n_q, const uint16_t* K, const uint16_t* V,
                                         int64_t n_kv, int32_t heads, int32_t head_dim, float scale, int32_t splits,
                                         void* O, int32_t out_fp32, float* lse, void* ws, size_t ws_bytes,
                                         void* stream) {
    if (heads < 1 || n_q < 1 || n_kv < 1) return ZB_ERR_SHAPE;
    if (head_dim != mrg::HD) return ZB_ERR_UNSUPPORTED;
    if (splits < 1 || splits > mrg::MAX_SPLITS || n_kv % splits != 0) return ZB_ERR_SHAPE;
    if (!Q || !K || !V || !O) return ZB_ERR_NULL;
    if (n_q > (1ll << 31) - 256 || n_kv > (1ll << 31) - 256) return ZB_ERR_UNSUPPORTED;
    if (!(scale > 0.f) || !isfinite(scale)) return ZB_ERR_SHAPE;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(lse) || !aligned16(ws))
        return ZB_ERR_ALIGN;
    if (splits == 1) return zb_dense_attn(Q, n_q, K, V, n_kv, heads, head_dim, scale, O, out_fp32, lse, stream);
    const mrg::Layout l = mrg::layout(n_q, heads, splits);
    if (!ws || ws_bytes < l.total) return ZB_ERR_WORKSPACE;
    DeviceInfo dev;
    zb_status e = current_device(&dev);
    if (e != ZB_OK) return e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(ws);
    uint16_t* qrep = reinterpret_cast<uint16_t*>(base + l.qrep);
    float* op = reinterpret_cast<float*>(base + l.op);
    float* lsep = reinterpret_cast<float*>(base + l.lsep);
    // queries of head h repeated for each of its virtual heads: [H][S][n_q][d]
    const size_t row_bytes = static_cast<size_t>(n_q) * mrg::HD * 2;
    for (int p = 0; p < splits; ++p) {
        if (cudaMemcpy2DAsync(qrep + static_cast<size_t>(p) * n_q * mrg::HD, row_bytes * splits, Q, row_bytes,
                              row_bytes, static_cast<size_t>(heads), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return ZB_ERR_CUDA;
    }
    e = zb_dense_attn(qrep, n_q, K, V, n_kv / splits, heads * splits, head_dim, scale, op, 1, lsep, stream);
    if (e != ZB_OK) return e;
    const long long warps = static_cast<long long>(heads) * n_q;
    const long long grid = (warps + mrg::THREADS / 32 - 1) / (mrg::THREADS / 32);
    if (grid > 0x7FFFFFFFll) return ZB_ERR_UNSUPPORTED;
    mrg::merge_kernel<<<static_cast<unsigned>(grid), mrg::THREADS, 0, st>>>(op, lsep, heads, splits, n_q, O,
                                                                          out_fp32 ? 1 : 0, lse);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}
