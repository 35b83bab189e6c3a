// Landmark pass: per-tile means of Q, K and V, and a whole-tile gather.
//
// "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D Reconstruction",
// Figure 1 (a) caption: an omitted key tile becomes one landmark whose key is
// the tile's mean key and whose value is its mean value.  The mean query of a
// tile is the pooled query used to score tile pairs.
//
// HBM-bound stream: a tile of one tensor is one contiguous run of n_j rows x
// 128 bytes, read by one warp with 16-byte loads and summed exactly (fp64, or
// fp32 where four values span few enough binades; exact for bf16 inputs unless
// a tile spans > ~38 binades), then divided by n_j.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace lmk {

constexpr int THREADS = 256;      // gather kernel
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

// Landmark kernel: one warp per (head, tile, tensor).  Lane l reads the
// 16-byte feature group l % 8 (columns 8 (l % 8) ..) of rows l / 8 + 4 m,
// m = 0..31, eight loads in flight, and sums each column exactly: four rows at
// a time in fp32 when their exponents span at most 14 binades (then every
// partial sum is a multiple of the smallest value's unit 2^(E-7) below 2^24 of
// them), else in fp64; quads are added in fp64.  A butterfly over the four row
// lanes of a feature group (xor 8, 16) leaves the exact column sums in every
// lane; lanes 0..7 write the means.  No shared memory and no barriers, so many
// warps per SM keep the loads in flight.
constexpr int LW_THREADS = 256;

ZB_DEVINL double quad_sum_lo(uint32_t a, uint32_t b, uint32_t c, uint32_t d, bool ok) {
    if (ok) return static_cast<double>((bf16_lo(a) + bf16_lo(b)) + (bf16_lo(c) + bf16_lo(d)));
    return (static_cast<double>(bf16_lo(a)) + static_cast<double>(bf16_lo(b))) +
           (static_cast<double>(bf16_lo(c)) + static_cast<double>(bf16_lo(d)));
}
ZB_DEVINL double quad_sum_hi(uint32_t a, uint32_t b, uint32_t c, uint32_t d, bool ok) {
    if (ok) return static_cast<double>((bf16_hi(a) + bf16_hi(b)) + (bf16_hi(c) + bf16_hi(d)));
    return (static_cast<double>(bf16_hi(a)) + static_cast<double>(bf16_hi(b))) +
           (static_cast<double>(bf16_hi(c)) + static_cast<double>(bf16_hi(d)));
}

__global__ void __launch_bounds__(LW_THREADS)
landmark_kernel(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ K,
                const uint16_t* __restrict__ V, int heads, long long N, int tile, int T,
                double* __restrict__ Qbar, double* __restrict__ Kbar, uint16_t* __restrict__ Kb16,
                uint16_t* __restrict__ Vb16) {
    const int lane = threadIdx.x & 31;
    const bool do_q = Q != nullptr;
    const int nt = do_q ? 3 : 2;
    const long long gw = static_cast<long long>(blockIdx.x) * (LW_THREADS / 32) + (threadIdx.x >> 5);
    const long long items = static_cast<long long>(heads) * T;
    if (gw >= items * nt) return;
    const long long item = gw / nt;
    const int t = (do_q ? 0 : 1) + static_cast<int>(gw % nt);  // 0 = Q, 1 = K, 2 = V
    const int h = static_cast<int>(item / T), j = static_cast<int>(item % T);
    const int n = static_cast<int>(min(static_cast<long long>(tile), N - static_cast<long long>(j) * tile));
    const uint16_t* X = t == 0 ? Q : (t == 1 ? K : V);
    const int cg = lane & 7, rl = lane >> 3;
    const uint4* rows = reinterpret_cast<const uint4*>(X + (static_cast<long long>(h) * N + static_cast<long long>(j) * tile) * HD);
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll 1
    for (int m0 = 0; m0 < 32; m0 += 8) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int r = rl + 4 * (m0 + u);
            v[u] = r < n ? rows[r * 8 + cg] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint4* w = v + 4 * q;
            const uint32_t x[4][4] = {{w[0].x, w[0].y, w[0].z, w[0].w}, {w[1].x, w[1].y, w[1].z, w[1].w},
                                      {w[2].x, w[2].y, w[2].z, w[2].w}, {w[3].x, w[3].y, w[3].z, w[3].w}};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                uint32_t mx = x[0][e] & 0x7FFF7FFFu, mn = mx;
#pragma unroll
                for (int r = 1; r < 4; ++r) {
                    const uint32_t mg = x[r][e] & 0x7FFF7FFFu;
                    asm("max.u16x2 %0, %0, %1;" : "+r"(mx) : "r"(mg));
                    asm("min.u16x2 %0, %0, %1;" : "+r"(mn) : "r"(mg));
                }
                const int lo_min = (mn >> 7) & 0xFF, lo_max = (mx >> 7) & 0xFF;
                const int hi_min = (mn >> 23) & 0xFF, hi_max = (mx >> 23) & 0xFF;
                const bool lo_ok = lo_min > 0 && lo_max - lo_min <= 14;
                const bool hi_ok = hi_min > 0 && hi_max - hi_min <= 14;
                if (lo_ok && hi_ok) {
                    // both columns exact in fp32: one packed fp32x2 chain (the same
                    // additions in the same order as quad_sum_lo / quad_sum_hi)
                    const uint64_t ab = f2_add(f2_pack(bf16_lo(x[0][e]), bf16_hi(x[0][e])),
                                               f2_pack(bf16_lo(x[1][e]), bf16_hi(x[1][e])));
                    const uint64_t cd = f2_add(f2_pack(bf16_lo(x[2][e]), bf16_hi(x[2][e])),
                                               f2_pack(bf16_lo(x[3][e]), bf16_hi(x[3][e])));
                    float slo, shi;
                    f2_unpack(f2_add(ab, cd), slo, shi);
                    acc[2 * e] += static_cast<double>(slo);
                    acc[2 * e + 1] += static_cast<double>(shi);
                } else {
                    acc[2 * e] += quad_sum_lo(x[0][e], x[1][e], x[2][e], x[3][e], lo_ok);
                    acc[2 * e + 1] += quad_sum_hi(x[0][e], x[1][e], x[2][e], x[3][e], hi_ok);
                }
            }
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 8);
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    }
    if (lane < 8) {
        const long long o = (static_cast<long long>(h) * T + j) * HD + 8 * cg;
        double mean[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)  // n = 128 or 64 is a power of two: the product by 1 / n is the exact quotient
            mean[e] = n == 128 ? acc[e] * 0.0078125 : (n == 64 ? acc[e] * 0.015625 : acc[e] / static_cast<double>(n));
        if (t == 0 || t == 1) {
            double2* dst = reinterpret_cast<double2*>((t == 0 ? Qbar : Kbar) + o);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_double2(mean[2 * e], mean[2 * e + 1]);
        }
        if (t == 1 || t == 2) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                pk[e] = static_cast<uint32_t>(f64_to_bf16_rne(mean[2 * e])) |
                        (static_cast<uint32_t>(f64_to_bf16_rne(mean[2 * e + 1])) << 16);
            *reinterpret_cast<uint4*>((t == 1 ? Kb16 : Vb16) + o) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
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
    const long long warps = static_cast<long long>(s.heads) * T * (Q ? 3 : 2);
    const long long grid = (warps + lmk::LW_THREADS / 32 - 1) / (lmk::LW_THREADS / 32);
    if (grid > 0x7FFFFFFFll) return ZB_ERR_UNSUPPORTED;
    lmk::landmark_kernel<<<static_cast<unsigned>(grid), lmk::LW_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
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
