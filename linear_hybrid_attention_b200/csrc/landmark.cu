// Landmark pass: per-tile means of Q, K and V, and a whole-tile gather.
//
// "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D Reconstruction",
// Figure 1 (a) caption: an omitted key tile becomes one landmark whose key is
// the tile's mean key and whose value is its mean value.  The mean query of a
// tile is the pooled query used to score tile pairs.
//
// HBM-bound stream: each CTA walks (head, tile) pairs; a tile of one tensor is
// one contiguous run of n_j rows x 128 bytes, read with 16-byte loads (thread
// t holds column group t % 8 of rows t / 8, t / 8 + 32, ...), summed in fp64
// (exact for bf16 inputs unless a tile spans > ~38 binades), reduced in a
// fixed order, divided by n_j.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace lmk {

constexpr int THREADS = 256;      // gather kernel
constexpr int LM_THREADS = 512;   // landmark kernel: 16 warps, 8 rows each
constexpr int HD = 64;

__device__ __forceinline__ void add8(double (&acc)[8], const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc[2 * e] += static_cast<double>(bf16_lo(w[e]));
        acc[2 * e + 1] += static_cast<double>(bf16_hi(w[e]));
    }
}

// Round-to-nearest-even of an fp64 value to bf16 bits, as one rounding: keep
// the top 8 significant bits of the double's significand (ties to even), then
// narrow to fp32, which is exact for values in fp32's normal range.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
    const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
    const unsigned long long low_mask = (1ull << 45) - 1;  // 52 - 7 dropped mantissa bits
    const unsigned long long low = u & low_mask;
    const unsigned long long half = 1ull << 44;
    unsigned long long t = u & ~low_mask;
    if (low > half || (low == half && ((t >> 45) & 1ull))) t += 1ull << 45;
    const float f = static_cast<float>(__longlong_as_double(static_cast<long long>(t)));
    return static_cast<uint16_t>(__float_as_uint(f) >> 16);
}

// Persistent landmark kernel: one CTA per SM walks (head, tile) items
// round-robin.  Thread 0 copies the Q, K, V runs of an item (n_j rows x 128 B
// each, contiguous) into a LM_STAGES-deep shared-memory ring with bulk copies;
// warp w sums rows [8 w, 8 w + 8) of each tensor, lane l columns 2l, 2l+1,
// in fp64 (exact for bf16 inputs unless a tile spans > ~38 binades); the 16
// warp partials are added in a fixed order by 192 threads, one output each.
// 16 warps per SM hide the latency of the fp32 -> fp64 conversions.
constexpr int LM_STAGES = 3;
constexpr uint32_t RUN_BYTES = 128 * HD * 2;  // one full tile of one tensor

struct LmSmem {
    uint8_t buf[LM_STAGES][3][RUN_BYTES];
    double part[2][LM_THREADS / 32][3][HD];
    uint64_t full[LM_STAGES];
    int abort_flag;
};

__global__ void __launch_bounds__(LM_THREADS, 1)
landmark_kernel(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ K,
                const uint16_t* __restrict__ V, int heads, long long N, int tile, int T,
                double* __restrict__ Qbar, double* __restrict__ Kbar, uint16_t* __restrict__ Kb16,
                uint16_t* __restrict__ Vb16, int* status, unsigned long long timeout_ns) {
    extern __shared__ uint8_t smem_raw[];
    LmSmem& sm = *reinterpret_cast<LmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool do_q = Q != nullptr;
    const int nt = do_q ? 3 : 2;         // tensors copied per item
    const int t0 = do_q ? 0 : 1;         // first tensor slot used (0 = Q, 1 = K, 2 = V)
    const long long total = static_cast<long long>(heads) * T;
    const long long first = blockIdx.x;
    const int cnt = first < total ? static_cast<int>((total - 1 - first) / gridDim.x + 1) : 0;
    const WaitCtx wc{status, &sm.abort_flag, timeout_ns};
    if (tid == 0) {
        sm.abort_flag = 0;
        for (int s = 0; s < LM_STAGES; ++s) mbar_init(smem_addr(&sm.full[s]), 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto item_of = [&](int it, int& h, int& j, int& n) {
        const long long w = first + static_cast<long long>(it) * gridDim.x;
        h = static_cast<int>(w / T);
        j = static_cast<int>(w % T);
        n = static_cast<int>(min(static_cast<long long>(tile), N - static_cast<long long>(j) * tile));
    };
    auto issue = [&](int it) {
        int h, j, n;
        item_of(it, h, j, n);
        const int s = it % LM_STAGES;
        const uint32_t bar = smem_addr(&sm.full[s]);
        const uint32_t bytes = static_cast<uint32_t>(n) * HD * 2;
        const long long off = (static_cast<long long>(h) * N + static_cast<long long>(j) * tile) * HD;
        mbar_arrive_expect_tx(bar, bytes * nt);
        if (do_q) bulk_load(smem_addr(sm.buf[s][0]), Q + off, bytes, bar);
        bulk_load(smem_addr(sm.buf[s][1]), K + off, bytes, bar);
        bulk_load(smem_addr(sm.buf[s][2]), V + off, bytes, bar);
    };
    int issued = 0;
    if (tid == 0)
        for (int it = 0; it < LM_STAGES && it < cnt; ++it) issue(it), ++issued;

    int consumed = 0;
    for (int it = 0; it < cnt; ++it) {
        const int s = it % LM_STAGES;
        int h, j, n;
        item_of(it, h, j, n);
        const bool good = mbar_wait(smem_addr(&sm.full[s]), (it / LM_STAGES) & 1, wc);
        if (good) consumed = it + 1;
        const int r0 = warp * 8;
        const int rows = good ? max(0, min(8, n - r0)) : 0;
#pragma unroll
        for (int t = 0; t < 3; ++t) {
            double a0 = 0.0, a1 = 0.0;
            if (t >= t0) {
                const uint32_t* src = reinterpret_cast<const uint32_t*>(sm.buf[s][t]) + r0 * (HD / 2) + lane;
                if (rows == 8) {
                    // all loads first, then a tree of adds (sums are exact, order-free)
                    uint32_t wv[8];
#pragma unroll
                    for (int r = 0; r < 8; ++r) wv[r] = src[r * (HD / 2)];
                    double l[4], h[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        l[r] = static_cast<double>(bf16_lo(wv[2 * r])) + static_cast<double>(bf16_lo(wv[2 * r + 1]));
                        h[r] = static_cast<double>(bf16_hi(wv[2 * r])) + static_cast<double>(bf16_hi(wv[2 * r + 1]));
                    }
                    a0 = (l[0] + l[1]) + (l[2] + l[3]);
                    a1 = (h[0] + h[1]) + (h[2] + h[3]);
                } else {
                    for (int r = 0; r < rows; ++r) {
                        const uint32_t wv = src[r * (HD / 2)];
                        a0 += static_cast<double>(bf16_lo(wv));
                        a1 += static_cast<double>(bf16_hi(wv));
                    }
                }
            }
            sm.part[it & 1][warp][t][2 * lane] = a0;
            sm.part[it & 1][warp][t][2 * lane + 1] = a1;
        }
        fence_proxy_async_smem();  // our reads of buf[s] precede the next bulk write into it
        if (__syncthreads_or(!good)) break;
        if (tid == 0 && it + LM_STAGES < cnt) issue(it + LM_STAGES), ++issued;
        if (tid < 3 * HD) {
            const int t = tid / HD, col = tid % HD;
            if (t >= t0) {
                double acc = 0.0;
#pragma unroll
                for (int wp = 0; wp < LM_THREADS / 32; ++wp) acc += sm.part[it & 1][wp][t][col];
                const double mean = acc / static_cast<double>(n);
                const long long o = (static_cast<long long>(h) * T + j) * HD + col;
                if (t == 0) {
                    Qbar[o] = mean;
                } else if (t == 1) {
                    Kbar[o] = mean;
                    Kb16[o] = f64_to_bf16_rne(mean);
                } else {
                    Vb16[o] = f64_to_bf16_rne(mean);
                }
            }
        }
    }
    // leave no bulk copy in flight
    if (tid == 0) {
        volatile int no_abort = 0;
        const WaitCtx w2{status, &no_abort, timeout_ns};
        for (int q = consumed; q < issued; ++q)
            mbar_wait(smem_addr(&sm.full[q % LM_STAGES]), (q / LM_STAGES) & 1, w2);
    }
}

__global__ void __launch_bounds__(THREADS)
gather_tiles_kernel(const uint16_t* __restrict__ X, int heads, long long N, int tile, int T,
                    const int32_t* __restrict__ tiles, int n_tiles, uint16_t* __restrict__ out,
                    int* status) {
    // one CTA per (head, listed tile); 16-byte copies, zero rows past N
    const long long w = blockIdx.x;
    const int h = static_cast<int>(w / n_tiles);
    const int m = static_cast<int>(w % n_tiles);
    int j = tiles[m];
    const bool bad = j < 0 || j >= T;
    if (bad && threadIdx.x == 0) flag_status(status, ZB_ERR_INDEX);
    const long long r0 = static_cast<long long>(j) * tile;
    const int per_row = HD / 8;  // uint4 per row
    const long long out_rows = static_cast<long long>(n_tiles) * tile;
    for (int e = threadIdx.x; e < tile * per_row; e += THREADS) {
        const int r = e / per_row, c = e % per_row;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (!bad && r0 + r < N)
            v = __ldg(reinterpret_cast<const uint4*>(X + ((static_cast<long long>(h) * N + r0 + r) * HD)) + c);
        reinterpret_cast<uint4*>(out + (static_cast<long long>(h) * out_rows + static_cast<long long>(m) * tile + r) * HD)[c] = v;
    }
}

}  // namespace lmk
}  // namespace zb

using namespace zb;

extern "C" zb_status zb_landmark_build(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                       zb_shape s, double* Qbar, double* Kbar,
                                       uint16_t* Kbar_bf16, uint16_t* Vbar_bf16, void* stream) {
    zb_status e = check_shape(s);
    if (e != ZB_OK) return e;
    if (!K || !V || !Kbar || !Kbar_bf16 || !Vbar_bf16) return ZB_ERR_NULL;
    if ((Q == nullptr) != (Qbar == nullptr)) return ZB_ERR_NULL;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Qbar) || !aligned16(Kbar) ||
        !aligned16(Kbar_bf16) || !aligned16(Vbar_bf16))
        return ZB_ERR_ALIGN;
    DeviceInfo dev;
    if ((e = current_device(&dev)) != ZB_OK) return e;
    const int T = static_cast<int>(n_tiles(s));
    const long long total = static_cast<long long>(s.heads) * T;
    const long long grid = total < dev.sm_count ? total : dev.sm_count;
    const size_t smem = sizeof(lmk::LmSmem) + 128;
    if (cudaFuncSetAttribute(lmk::landmark_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return ZB_ERR_CUDA;
    lmk::landmark_kernel<<<static_cast<unsigned>(grid), lmk::LM_THREADS, smem, static_cast<cudaStream_t>(stream)>>>(
        Q, K, V, s.heads, s.n_tokens, s.tile, T, Qbar, Kbar, Kbar_bf16, Vbar_bf16, dev.status,
        wait_timeout_ns());
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}

extern "C" zb_status zb_gather_tiles(const uint16_t* X, zb_shape s, const int32_t* tiles,
                                     int32_t n_tiles_, uint16_t* out, void* stream) {
    zb_status e = check_shape(s);
    if (e != ZB_OK) return e;
    if (!X || !tiles || !out) return ZB_ERR_NULL;
    if (n_tiles_ < 1) return ZB_ERR_SHAPE;
    if (!aligned16(X) || !aligned16(out)) return ZB_ERR_ALIGN;
    DeviceInfo dev;
    if ((e = current_device(&dev)) != ZB_OK) return e;
    const long long grid = static_cast<long long>(s.heads) * n_tiles_;
    if (grid > 0x7FFFFFFFll) return ZB_ERR_UNSUPPORTED;
    lmk::gather_tiles_kernel<<<static_cast<unsigned>(grid), lmk::THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
        X, s.heads, s.n_tokens, s.tile, static_cast<int>(n_tiles(s)), tiles, n_tiles_, out, dev.status);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}
