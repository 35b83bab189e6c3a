// Tile selection: fp64 scores of every (query tile, key tile) pair from the
// mean-pooled tiles, then the k largest per query tile.
//
// "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D Reconstruction",
// Figure 1 (a) caption names "selected tiles"; the pages give no criterion.
// Reading used: score(i, j) = Qbar_i . Kbar_j in fp64, the k largest kept,
// equal scores resolved toward the lower key-tile index, output ascending.
//
// One CTA scores R query tiles of one head against all T key tiles (scores
// kept in shared memory as fp64), then, row by row, finds the k-th largest
// score with an 8-bit-digit radix select on order-preserving 64-bit keys, and
// writes the kept indices in ascending order with block-wide prefix sums.
#include <cuda_runtime.h>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace topk {

constexpr int THREADS = 256;
constexpr int HD = 64;
constexpr size_t SCORE_SMEM_BUDGET = 200 * 1024;
constexpr int MAX_ROWS = 32;

// Order-preserving map of an fp64 value to uint64 (larger value -> larger key);
// -0.0 is folded onto +0.0 so that they tie.
__device__ __forceinline__ unsigned long long order_key(double s) {
    if (s == 0.0) s = 0.0;
    const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(s));
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// Block-wide exclusive prefix sum of one int per thread; returns the exclusive
// value, writes the block total to *total.  Uses `scratch` (>= THREADS/32 ints).
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    int wsum = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < THREADS / 32; ++w) {
        const int s = scratch[w];
        if (w < warp) wsum += s;
        tot += s;
    }
    __syncthreads();
    *total = tot;
    return wsum + x - v;
}

__global__ void __launch_bounds__(THREADS)
score_topk_kernel(const double* __restrict__ Qbar, const double* __restrict__ Kbar, int heads,
                  int T, int k, int rows_per_cta, int32_t* __restrict__ idx) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    double* qs = reinterpret_cast<double*>(smem_raw);                 // [R][64]
    double* sc = qs + static_cast<size_t>(rows_per_cta) * HD;        // [R][T]
    __shared__ unsigned int hist[256];
    __shared__ int scan_scratch[THREADS / 32];
    __shared__ int sel_bucket, sel_above;

    const int tid = threadIdx.x;
    const int blocks_per_head = (T + rows_per_cta - 1) / rows_per_cta;
    const int h = blockIdx.x / blocks_per_head;
    const int i0 = (blockIdx.x % blocks_per_head) * rows_per_cta;
    const int R = min(rows_per_cta, T - i0);
    const double* qh = Qbar + (static_cast<long long>(h) * T + i0) * HD;
    const double* kh = Kbar + static_cast<long long>(h) * T * HD;

    for (int e = tid; e < R * HD; e += THREADS) qs[e] = qh[e];
    __syncthreads();

    // ---- scores: thread owns key tiles j = tid, tid + 256, ...; fp64 FMA chain over d
    for (int j = tid; j < T; j += THREADS) {
        double acc[MAX_ROWS];
#pragma unroll
        for (int r = 0; r < MAX_ROWS; ++r) acc[r] = 0.0;
        const double2* kj = reinterpret_cast<const double2*>(kh + static_cast<long long>(j) * HD);
#pragma unroll 4
        for (int c2 = 0; c2 < HD / 2; ++c2) {
            const double2 kv = __ldg(kj + c2);
#pragma unroll
            for (int r = 0; r < MAX_ROWS; ++r) {
                if (r < R) {
                    const double2 qv = reinterpret_cast<const double2*>(qs + r * HD)[c2];
                    acc[r] = fma(qv.x, kv.x, acc[r]);
                    acc[r] = fma(qv.y, kv.y, acc[r]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < MAX_ROWS; ++r)
            if (r < R) sc[static_cast<size_t>(r) * T + j] = acc[r];
    }
    __syncthreads();

    for (int r = 0; r < R; ++r) {
        const double* row = sc + static_cast<size_t>(r) * T;
        int32_t* out = idx + (static_cast<long long>(h) * T + i0 + r) * static_cast<long long>(k);
        if (k == 0) continue;
        if (k == T) {
            for (int j = tid; j < T; j += THREADS) out[j] = j;
            continue;
        }
        // ---- radix select of the k-th largest key, 8 bits per pass from the top
        unsigned long long prefix = 0, mask = 0;
        int need = k;
        for (int shift = 56; shift >= 0; shift -= 8) {
            for (int b = tid; b < 256; b += THREADS) hist[b] = 0u;
            __syncthreads();
            // uniform trip count: every lane reaches the warp-collective calls
            for (int j0 = 0; j0 < T; j0 += THREADS) {
                const int j = j0 + tid;
                const unsigned long long key = j < T ? order_key(row[j]) : 0ull;
                const bool m = j < T && (key & mask) == prefix;
                const unsigned int digit = static_cast<unsigned int>((key >> shift) & 0xFFu);
                const unsigned int active = __ballot_sync(0xffffffffu, m);
                if (m) {
                    const unsigned int peers = __match_any_sync(active, digit);
                    if ((__ffs(peers) - 1) == (tid & 31)) atomicAdd(&hist[digit], __popc(peers));
                }
            }
            __syncthreads();
            if (tid < 32) {
                // lane l owns bins 8l..8l+7; find the bin holding the need-th largest
                unsigned int c[8], lsum = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) lsum += (c[e] = hist[tid * 8 + e]);
                // inclusive suffix sum over lanes: x = sum of lanes >= tid
                unsigned int x = lsum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned int y = __shfl_down_sync(0xffffffffu, x, o);
                    if (tid + o < 32) x += y;
                }
                const unsigned int suffix = x - lsum;  // sum of lanes > tid
                if (suffix < static_cast<unsigned int>(need) && suffix + lsum >= static_cast<unsigned int>(need)) {
                    unsigned int run = suffix;
                    for (int e = 7; e >= 0; --e) {
                        if (run + c[e] >= static_cast<unsigned int>(need)) {
                            sel_bucket = tid * 8 + e;
                            sel_above = static_cast<int>(run);
                            break;
                        }
                        run += c[e];
                    }
                }
            }
            __syncthreads();
            const int bsel = sel_bucket;
            need -= sel_above;
            prefix |= static_cast<unsigned long long>(bsel) << shift;
            mask |= 0xFFull << shift;
            const bool done = static_cast<int>(hist[bsel]) == need;
            __syncthreads();
            if (done) break;
        }
        // ---- write kept indices ascending: keys above the prefix, plus the
        // first `need` (lowest j) keys equal to it
        int run_eq = 0, run_sel = 0;
        for (int j0 = 0; j0 < T; j0 += THREADS) {
            const int j = j0 + tid;
            bool gt = false, eq = false;
            if (j < T) {
                const unsigned long long km = order_key(row[j]) & mask;
                gt = km > prefix;
                eq = km == prefix;
            }
            int tot_eq;
            const int eq_rank = run_eq + block_excl_scan(eq ? 1 : 0, scan_scratch, &tot_eq);
            const bool sel = gt || (eq && eq_rank < need);
            int tot_sel;
            const int pos = run_sel + block_excl_scan(sel ? 1 : 0, scan_scratch, &tot_sel);
            if (sel) out[pos] = j;
            run_eq += tot_eq;
            run_sel += tot_sel;
        }
        __syncthreads();
    }
}

}  // namespace topk
}  // namespace zb

using namespace zb;

extern "C" zb_status zb_tile_score_topk(const double* Qbar, const double* Kbar, zb_shape s,
                                        int32_t k, int32_t* idx, void* stream) {
    zb_status e = check_shape(s);
    if (e != ZB_OK) return e;
    if (!Qbar || !Kbar || (!idx && k > 0)) return ZB_ERR_NULL;
    const long long T = n_tiles(s);
    if (T > 32768) return ZB_ERR_UNSUPPORTED;
    if (k < 0 || k > T) return ZB_ERR_SHAPE;
    if (!aligned16(Qbar) || !aligned16(Kbar) || !aligned16(idx)) return ZB_ERR_ALIGN;
    if (k == 0) return ZB_OK;
    DeviceInfo dev;
    if ((e = current_device(&dev)) != ZB_OK) return e;
    long long R = static_cast<long long>(topk::SCORE_SMEM_BUDGET / (static_cast<size_t>(T) * 8 + 64 * 8));
    if (R > topk::MAX_ROWS) R = topk::MAX_ROWS;
    if (R > T) R = T;
    if (R < 1) return ZB_ERR_UNSUPPORTED;
    const size_t smem = static_cast<size_t>(R) * (static_cast<size_t>(T) + 64) * 8;
    if (cudaFuncSetAttribute(topk::score_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return ZB_ERR_CUDA;
    const long long grid = static_cast<long long>(s.heads) * ((T + R - 1) / R);
    if (grid > 0x7FFFFFFFll) return ZB_ERR_UNSUPPORTED;
    topk::score_topk_kernel<<<static_cast<unsigned>(grid), topk::THREADS, smem, static_cast<cudaStream_t>(stream)>>>(
        Qbar, Kbar, s.heads, static_cast<int>(T), k, static_cast<int>(R), idx);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}
