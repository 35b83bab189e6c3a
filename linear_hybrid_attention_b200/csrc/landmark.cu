// Landmark pass: per-tile means of Q, K and V, and a whole-tile gather.
//
// "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D Reconstruction",
// Figure 1 (a) caption: an omitted key tile becomes one landmark whose key is
// the tile's mean key and whose value is its mean value.  The mean query of a
// tile is the pooled query used to score tile pairs.
//
// HBM-bound stream: each CTA walks (head, tile) pairs; a tile of one tensor is
// one contiguous run of n_j rows x 128 bytes, staged in shared memory by bulk
// copies, summed in fp64 (exact for bf16 inputs unless a tile spans > ~38
// binades), reduced in a fixed order, divided by n_j.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace lmk {

constexpr int THREADS = 256;      // gather kernel
constexpr int LM_THREADS = 544;   // landmark kernel: 16 compute warps (8 rows each) + a producer warp
constexpr int HD = 64;

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
// round-robin, with roles that meet only at mbarriers (no CTA-wide barrier per
// tile):
//   warp 16 (one lane)  copies the Q, K, V runs of an item (n_j rows x 128 B
//                       each, contiguous) into a LM_STAGES-deep ring with bulk
//                       copies, once the 16 compute warps have read the stage;
//   warps 0..15         warp w sums rows [8 w, 8 w + 8) of each tensor, lane l
//                       columns 2l, 2l+1, in fp64 (exact for bf16 inputs unless
//                       a tile spans > ~38 binades), into one of three
//                       partial tables; warps 0..5 (192 threads, one output
//                       each) then add the 16 partials of the item as a fixed
//                       4-level tree and write the means, while the other
//                       warps already sum the next items.
// 16 compute warps per SM hide the latency of the fp32 -> fp64 conversions.
constexpr int LM_STAGES = 3;
constexpr int NPB = 3;        // partial tables: the compute warps run up to two items ahead of the reduction
constexpr int LM_WARPS = 16;  // compute warps
static_assert(LM_WARPS == 16, "the partial reduction is a tree over 16 warps");
constexpr uint32_t RUN_BYTES = 128 * HD * 2;  // one full tile of one tensor

struct LmSmem {
    uint8_t buf[LM_STAGES][3][RUN_BYTES];
    double part[NPB][LM_WARPS][3][HD];
    uint64_t full[LM_STAGES], empty[LM_STAGES];
    uint64_t pfull[NPB], pempty[NPB];
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
        for (int s = 0; s < LM_STAGES; ++s) {
            mbar_init(smem_addr(&sm.full[s]), 1);
            mbar_init(smem_addr(&sm.empty[s]), LM_WARPS);
        }
        for (int b = 0; b < NPB; ++b) {
            mbar_init(smem_addr(&sm.pfull[b]), LM_WARPS);
            mbar_init(smem_addr(&sm.pempty[b]), 3 * HD);
        }
        fence_mbar_init();
    }
    __syncthreads();

    auto item_of = [&](int it, int& h, int& j, int& n) {
        const long long w = first + static_cast<long long>(it) * gridDim.x;
        h = static_cast<int>(w / T);
        j = static_cast<int>(w % T);
        n = static_cast<int>(min(static_cast<long long>(tile), N - static_cast<long long>(j) * tile));
    };

    if (warp == LM_WARPS) {
        if (lane == 0) {
            // ================================================= producer ====
            uint32_t issued_mask = 0, par_mask = 0;
            for (int it = 0; it < cnt; ++it) {
                const int s = it % LM_STAGES;
                const uint32_t use = static_cast<uint32_t>(it / LM_STAGES);
                if (!mbar_wait_sleep(smem_addr(&sm.empty[s]), (use & 1) ^ 1, wc, 20000)) break;
                int h, j, n;
                item_of(it, h, j, n);
                const uint32_t bar = smem_addr(&sm.full[s]);
                const uint32_t bytes = static_cast<uint32_t>(n) * HD * 2;
                const long long off = (static_cast<long long>(h) * N + static_cast<long long>(j) * tile) * HD;
                mbar_arrive_expect_tx(bar, bytes * nt);
                if (do_q) bulk_load(smem_addr(sm.buf[s][0]), Q + off, bytes, bar);
                bulk_load(smem_addr(sm.buf[s][1]), K + off, bytes, bar);
                bulk_load(smem_addr(sm.buf[s][2]), V + off, bytes, bar);
                issued_mask |= 1u << s;
                par_mask = (par_mask & ~(1u << s)) | ((use & 1u) << s);
            }
            // leave no bulk copy in flight (bounded, even after an abort)
            volatile int no_abort = 0;
            const WaitCtx w2{status, &no_abort, drain_timeout_ns(timeout_ns)};
            for (int s = 0; s < LM_STAGES; ++s)
                if ((issued_mask >> s) & 1u) mbar_wait(smem_addr(&sm.full[s]), (par_mask >> s) & 1u, w2);
        }
        __syncwarp();
    } else {
        // ============================================ compute warps ====
        for (int it = 0; it < cnt; ++it) {
            const int s = it % LM_STAGES, pb = it % NPB;
            const uint32_t use = static_cast<uint32_t>(it / LM_STAGES), pu = static_cast<uint32_t>(it / NPB);
            int h, j, n;
            item_of(it, h, j, n);
            if (!mbar_wait_warp(smem_addr(&sm.full[s]), use & 1, wc)) break;
            const int r0 = warp * 8;
            const int rows = max(0, min(8, n - r0));
            double acc[3][2];
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
                        double l[4], hh[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            l[r] = static_cast<double>(bf16_lo(wv[2 * r])) + static_cast<double>(bf16_lo(wv[2 * r + 1]));
                            hh[r] = static_cast<double>(bf16_hi(wv[2 * r])) + static_cast<double>(bf16_hi(wv[2 * r + 1]));
                        }
                        a0 = (l[0] + l[1]) + (l[2] + l[3]);
                        a1 = (hh[0] + hh[1]) + (hh[2] + hh[3]);
                    } else {
                        for (int r = 0; r < rows; ++r) {
                            const uint32_t wv = src[r * (HD / 2)];
                            a0 += static_cast<double>(bf16_lo(wv));
                            a1 += static_cast<double>(bf16_hi(wv));
                        }
                    }
                }
                acc[t][0] = a0;
                acc[t][1] = a1;
            }
            // this warp is done with stage s
            fence_proxy_async_smem();  // our reads precede the next bulk write into it
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&sm.empty[s]));
            // partial table pb is free once the item NPB back was reduced
            if (!mbar_wait_warp(smem_addr(&sm.pempty[pb]), (pu & 1) ^ 1, wc)) break;
#pragma unroll
            for (int t = 0; t < 3; ++t) {
                sm.part[pb][warp][t][2 * lane] = acc[t][0];
                sm.part[pb][warp][t][2 * lane + 1] = acc[t][1];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&sm.pfull[pb]));
            if (tid < 3 * HD) {
                // fixed-order reduction of the 16 partials (a 4-level tree: the
                // partials and their sums are exact, so any fixed order gives the
                // same value), one output per thread
                if (!mbar_wait_warp(smem_addr(&sm.pfull[pb]), pu & 1, wc)) break;
                const int t = tid / HD, col = tid % HD;
                double v8[LM_WARPS / 2];
#pragma unroll
                for (int wp = 0; wp < LM_WARPS / 2; ++wp)
                    v8[wp] = sm.part[pb][2 * wp][t][col] + sm.part[pb][2 * wp + 1][t][col];
                const double sum = ((v8[0] + v8[1]) + (v8[2] + v8[3])) + ((v8[4] + v8[5]) + (v8[6] + v8[7]));
                mbar_arrive(smem_addr(&sm.pempty[pb]));
                if (t >= t0) {
                    // n = 128 or 64 is a power of two: the product by 1 / n is the exact quotient
                    const double mean = n == 128 ? sum * 0.0078125
                                                 : (n == 64 ? sum * 0.015625 : sum / static_cast<double>(n));
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
