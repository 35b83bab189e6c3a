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

constexpr int THREADS = 256;
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

__global__ void __launch_bounds__(THREADS)
landmark_kernel(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ K,
                const uint16_t* __restrict__ V, int heads, long long N, int tile, int T,
                double* __restrict__ Qbar, double* __restrict__ Kbar, uint16_t* __restrict__ Kb16,
                uint16_t* __restrict__ Vb16) {
    __shared__ double part[3][THREADS / 32][8][8];  // [tensor][warp][col group][col]
    const int tid = threadIdx.x;
    const int cg = tid & 7;          // 16-byte column group (8 columns)
    const int rs = tid >> 3;         // row slot 0..31
    const int warp = tid >> 5, lane = tid & 31;
    const bool do_q = Q != nullptr;
    const long long total = static_cast<long long>(heads) * T;
    for (long long w = blockIdx.x; w < total; w += gridDim.x) {
        const int h = static_cast<int>(w / T);
        const int j = static_cast<int>(w % T);
        const long long r0 = static_cast<long long>(j) * tile;
        const int n = static_cast<int>(min(static_cast<long long>(tile), N - r0));
        const long long base = (static_cast<long long>(h) * N + r0) * HD;
        double aq[8] = {0, 0, 0, 0, 0, 0, 0, 0}, ak[8] = {0, 0, 0, 0, 0, 0, 0, 0},
               av[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        // issue all loads of this thread first, then accumulate (memory-level parallelism)
        uint4 lq[4], lk[4], lv[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int r = rs + 32 * m;
            const bool in = r < n;
            const long long off = base + static_cast<long long>(r) * HD + cg * 8;
            lk[m] = in ? __ldg(reinterpret_cast<const uint4*>(K + off)) : make_uint4(0, 0, 0, 0);
            lv[m] = in ? __ldg(reinterpret_cast<const uint4*>(V + off)) : make_uint4(0, 0, 0, 0);
            lq[m] = (in && do_q) ? __ldg(reinterpret_cast<const uint4*>(Q + off)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            add8(ak, lk[m]);
            add8(av, lv[m]);
            if (do_q) add8(aq, lq[m]);
        }
        // reduce over the 4 row slots of this warp that share cg (lanes cg, cg+8, cg+16, cg+24)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
#pragma unroll
            for (int o = 8; o <= 16; o <<= 1) {
                ak[c] += __shfl_xor_sync(0xffffffffu, ak[c], o);
                av[c] += __shfl_xor_sync(0xffffffffu, av[c], o);
                aq[c] += __shfl_xor_sync(0xffffffffu, aq[c], o);
            }
        }
        if (lane < 8) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                part[0][warp][cg][c] = aq[c];
                part[1][warp][cg][c] = ak[c];
                part[2][warp][cg][c] = av[c];
            }
        }
        __syncthreads();
        if (tid < 3 * HD) {
            const int t = tid / HD;       // 0 = Q, 1 = K, 2 = V
            const int col = tid % HD;
            double s = 0.0;
#pragma unroll
            for (int wp = 0; wp < THREADS / 32; ++wp) s += part[t][wp][col >> 3][col & 7];
            const double mean = s / static_cast<double>(n);
            const long long o = (static_cast<long long>(h) * T + j) * HD + col;
            if (t == 0) {
                if (do_q) Qbar[o] = mean;
            } else if (t == 1) {
                Kbar[o] = mean;
                Kb16[o] = f64_to_bf16_rne(mean);
            } else {
                Vb16[o] = f64_to_bf16_rne(mean);
            }
        }
        __syncthreads();
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
    const long long grid = total < 8ll * dev.sm_count ? total : 8ll * dev.sm_count;
    lmk::landmark_kernel<<<static_cast<unsigned>(grid), lmk::THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
        Q, K, V, s.heads, s.n_tokens, s.tile, T, Qbar, Kbar, Kbar_bf16, Vbar_bf16);
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
