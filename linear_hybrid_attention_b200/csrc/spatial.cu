// Spatial tiles: a token order that groups each view's patches into 2-D
// windows, and the row gather that moves tensors into and out of that order.
//
// "3D reconstruction drops dense attention layer by layer: up to 5.6x
// end-to-end speedup at 1,024 views", synopsis: softmax is kept exact over
// selected *spatial* tiles.  Reading: a view is `specials` camera/register
// tokens followed by grid x grid patch tokens in row-major order; the spatial
// order keeps the specials first and then lists the patches window by window
// (win_rows x win_cols windows, row-major over the window grid, row-major
// inside a window, the windows at the right and bottom edges smaller).  The
// tile-sparse stage then runs unchanged on the reordered tokens, whose
// contiguous tiles cover compact 2-D regions, and each output row is moved
// back to its token's original position.
//
// zb_gather_rows is an HBM stream (one read and one write of every row): a
// warp moves 4 rows of 128 bytes per pass with 16-byte loads, lane l taking
// chunk l % 8 of row l / 8; the row index is read once per row.
#include <cuda_runtime.h>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace spat {

constexpr int THREADS = 256;
constexpr int HD = 64;

__global__ void __launch_bounds__(THREADS)
gather_rows_kernel(const uint4* __restrict__ X, long long n_in, long long n_out, int heads,
                   const int32_t* __restrict__ rows, uint4* __restrict__ out, int* status) {
    const long long total = static_cast<long long>(heads) * n_out;   // output rows
    const int chunk = threadIdx.x & 7;
    long long r = (static_cast<long long>(blockIdx.x) * THREADS + threadIdx.x) >> 3;
    const long long stride = (static_cast<long long>(gridDim.x) * THREADS) >> 3;
    int bad = 0;
    for (; r < total; r += stride) {
        const long long h = r / n_out, o = r - h * n_out;
        const int src = __ldg(rows + o);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (src >= 0 && src < n_in) v = __ldcs(X + (h * n_in + src) * (HD / 8) + chunk);
        else bad = 1;
        __stcs(out + r * (HD / 8) + chunk, v);
    }
    if (bad) flag_status(status, ZB_ERR_INDEX);
}

}  // namespace spat
}  // namespace zb

using namespace zb;

extern "C" zb_status zb_spatial_order(int32_t views, int32_t grid, int32_t specials, int32_t win_rows,
                                      int32_t win_cols, int32_t* order, int32_t* inverse) {
    if (views < 1 || grid < 1 || specials < 0 || win_rows < 1 || win_cols < 1) return ZB_ERR_SHAPE;
    if (!order) return ZB_ERR_NULL;
    const long long per_view = static_cast<long long>(specials) + static_cast<long long>(grid) * grid;
    if (per_view * views > 0x7FFFFFFFll) return ZB_ERR_UNSUPPORTED;
    long long p = 0;
    for (int v = 0; v < views; ++v) {
        const long long base = v * per_view;
        for (int t = 0; t < specials; ++t) order[p++] = static_cast<int32_t>(base + t);
        for (int wy = 0; wy < grid; wy += win_rows)
            for (int wx = 0; wx < grid; wx += win_cols) {
                const int ye = wy + win_rows < grid ? wy + win_rows : grid;
                const int xe = wx + win_cols < grid ? wx + win_cols : grid;
                for (int y = wy; y < ye; ++y)
                    for (int x = wx; x < xe; ++x)
                        order[p++] = static_cast<int32_t>(base + specials + static_cast<long long>(grid) * y + x);
            }
    }
    if (inverse)
        for (long long q = 0; q < p; ++q) inverse[order[q]] = static_cast<int32_t>(q);
    return ZB_OK;
}

extern "C" zb_status zb_gather_rows(const uint16_t* X, int32_t heads, int64_t n_in, int64_t n_out,
                                    int32_t head_dim, const int32_t* rows, uint16_t* out, void* stream) {
    if (heads < 1 || n_in < 1 || n_out < 1) return ZB_ERR_SHAPE;
    if (head_dim != 64) return ZB_ERR_UNSUPPORTED;
    if (n_in > 0x7FFFFFFFll || n_out > 0x7FFFFFFFll) return ZB_ERR_UNSUPPORTED;
    if (!X || !rows || !out) return ZB_ERR_NULL;
    if (!aligned16(X) || !aligned16(out) || (reinterpret_cast<uintptr_t>(rows) & 3u)) return ZB_ERR_ALIGN;
    DeviceInfo dev;
    zb_status e = current_device(&dev);
    if (e != ZB_OK) return e;
    const long long rows_total = static_cast<long long>(heads) * n_out;
    long long blocks = (rows_total * 8 + spat::THREADS - 1) / spat::THREADS;
    const long long cap = static_cast<long long>(dev.sm_count) * 8;   // 8 CTAs of 256 threads per SM
    if (blocks > cap) blocks = cap;
    spat::gather_rows_kernel<<<static_cast<unsigned>(blocks), spat::THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4*>(X), n_in, n_out, heads, rows, reinterpret_cast<uint4*>(out), dev.status);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}
