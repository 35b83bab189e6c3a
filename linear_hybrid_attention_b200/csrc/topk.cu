// Tile selection: fp64 scores of every (query tile, key tile) pair from the
// mean-pooled tiles, then the k largest per query tile.
//
// "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D Reconstruction",
// Figure 1 (a) caption names "selected tiles"; the pages give no criterion.
// Reading used: score(i, j) = Qbar_i . Kbar_j in fp64, the k largest kept,
// equal scores resolved toward the lower key-tile index, output ascending.
//
// Two kernels per group of heads (as many heads as the workspace holds):
//  * score_gemm_kernel: register-tiled fp64 GEMM, 128 x 128 scores per CTA,
//    8 x 8 per thread, full d = 64 staged (transposed) in shared memory; each
//    score is one FMA chain over d in index order.  Scores go to the workspace.
//  * select_kernel: one CTA per (head, query tile); the T scores become
//    order-preserving 64-bit keys in shared memory, the k-th largest is found
//    by a 12-bit-digit radix select (4,096-bin shared-memory histogram, early
//    exit once the bucket holds exactly the remaining count), and the kept
//    indices are written in ascending order with two block-wide prefix sums.
#include <cuda_runtime.h>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace topk {

constexpr int HD = 64;
constexpr int GT = 128;            // GEMM CTA tile (rows and columns)
constexpr int GTHREADS = 256;
constexpr int STHREADS = 512;
constexpr int MAX_T = 32768;
constexpr size_t SMEM_SCORE_LIMIT = 200 * 1024;  // scores kept in smem up to this size

// Order-preserving map of an fp64 value to uint64 (larger value -> larger key);
// -0.0 is folded onto +0.0 so that they tie.
__device__ __forceinline__ unsigned long long order_key(double s) {
    if (s == 0.0) s = 0.0;
    const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(s));
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// ------------------------------------------------------------- GEMM ----
// grid: (ceil(T/128) column blocks, ceil(T/128) row blocks, heads in group).
// Shared memory holds the 128-row blocks of Qbar and Kbar transposed, with a
// row stride of 129 doubles so that the transposing stores and the inner-loop
// reads are bank-conflict free; thread (ty, tx) owns rows ty + 16 a and
// columns tx + 16 b (a, b < 8), so a warp reads 16 consecutive doubles.
constexpr int GS = GT + 1;

__global__ void __launch_bounds__(GTHREADS)
score_gemm_kernel(const double* __restrict__ Qbar, const double* __restrict__ Kbar, int T, int h0,
                  double* __restrict__ scores) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    double* qt = reinterpret_cast<double*>(smem_raw);  // [64][129]
    double* kt = qt + HD * GS;                         // [64][129]
    const int h = h0 + blockIdx.z;
    const int i0 = blockIdx.y * GT, j0 = blockIdx.x * GT;
    const double* qh = Qbar + static_cast<long long>(h) * T * HD;
    const double* kh = Kbar + static_cast<long long>(h) * T * HD;
    for (int e = threadIdx.x; e < GT * HD; e += GTHREADS) {
        const int r = e / HD, c = e % HD;  // coalesced global reads
        qt[c * GS + r] = (i0 + r < T) ? qh[static_cast<long long>(i0 + r) * HD + c] : 0.0;
        kt[c * GS + r] = (j0 + r < T) ? kh[static_cast<long long>(j0 + r) * HD + c] : 0.0;
    }
    __syncthreads();
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    double acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.0;
#pragma unroll 2
    for (int c = 0; c < HD; ++c) {
        double qv[8], kv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            qv[u] = qt[c * GS + ty + 16 * u];
            kv[u] = kt[c * GS + tx + 16 * u];
        }
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int b = 0; b < 8; ++b) acc[a][b] = fma(qv[a], kv[b], acc[a][b]);
    }
    double* out = scores + static_cast<long long>(blockIdx.z) * T * T;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int i = i0 + ty + 16 * a;
        if (i >= T) continue;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int j = j0 + tx + 16 * b;
            if (j < T) out[static_cast<long long>(i) * T + j] = acc[a][b];
        }
    }
}

// Block-wide exclusive prefix sum of one int per thread (STHREADS threads).
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
    for (int w = 0; w < STHREADS / 32; ++w) {
        const int s = scratch[w];
        if (w < warp) wsum += s;
        tot += s;
    }
    __syncthreads();
    *total = tot;
    return wsum + x - v;
}

// Block-wide exclusive suffix sum (the sum over higher-numbered threads) of one
// int per thread (STHREADS threads).
__device__ __forceinline__ int block_excl_suffix(int v, int* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;  // inclusive suffix sum within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
    }
    if (lane == 0) scratch[warp] = x;
    __syncthreads();
    int above = 0;
#pragma unroll
    for (int w = 0; w < STHREADS / 32; ++w)
        if (w > warp) above += scratch[w];
    __syncthreads();
    return above + x - v;
}

// ----------------------------------------------------------- select ----
// grid: heads in group x T rows.  The row's scores become order keys in shared
// memory when they fit (`in_smem`), else they are read from the workspace on
// every pass.  Radix select of the k-th largest key from the top in 12-bit
// digits (4,096 bins, one shared-memory atomic per counted key); after each
// digit the bucket that holds the k-th key is found with a block-wide suffix
// sum, and the search stops as soon as that bucket holds exactly the keys
// still needed (usually after two digits: 24 bits of the key).
constexpr int DIGIT = 12;
constexpr int NBINS = 1 << DIGIT;
constexpr int BPT = NBINS / STHREADS;             // bins per thread
static_assert(BPT * STHREADS == NBINS, "bins per thread");

__global__ void __launch_bounds__(STHREADS)
select_kernel(const double* __restrict__ scores, int T, int k, int h0, int in_smem,
              int32_t* __restrict__ idx) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ unsigned int hist[NBINS];
    __shared__ int scan_scratch[STHREADS / 32];
    __shared__ int sel_bucket, sel_above;
    const int tid = threadIdx.x;
    const int hl = blockIdx.x / T, i = blockIdx.x % T;
    const double* grow = scores + (static_cast<long long>(hl) * T + i) * T;
    unsigned long long* skey = reinterpret_cast<unsigned long long*>(smem_raw);
    if (in_smem) {
        for (int j = tid; j < T; j += STHREADS) skey[j] = order_key(grow[j]);
        __syncthreads();
    }
    auto key_of = [&](int j) -> unsigned long long { return in_smem ? skey[j] : order_key(grow[j]); };
    int32_t* out = idx + (static_cast<long long>(h0 + hl) * T + i) * static_cast<long long>(k);

    unsigned long long prefix = 0, mask = 0;
    int need = k;
    for (int shift = 64 - DIGIT;; shift -= DIGIT) {
        const int sh = shift < 0 ? 0 : shift;
        const int width = shift < 0 ? shift + DIGIT : DIGIT;
        const unsigned int dmask = (1u << width) - 1u;
#pragma unroll
        for (int e = 0; e < BPT; ++e) hist[BPT * tid + e] = 0u;
        __syncthreads();
        for (int j = tid; j < T; j += STHREADS) {
            const unsigned long long key = key_of(j);
            if ((key & mask) == prefix) atomicAdd(&hist[static_cast<unsigned int>(key >> sh) & dmask], 1u);
        }
        __syncthreads();
        unsigned int c[BPT];
        int local = 0;
#pragma unroll
        for (int e = 0; e < BPT; ++e) local += static_cast<int>(c[e] = hist[BPT * tid + e]);
        const int above = block_excl_suffix(local, scan_scratch);
        if (above < need && above + local >= need) {
            int run = above;
#pragma unroll
            for (int e = BPT - 1; e >= 0; --e) {
                if (run + static_cast<int>(c[e]) >= need) {
                    sel_bucket = BPT * tid + e;
                    sel_above = run;
                    break;
                }
                run += static_cast<int>(c[e]);
            }
        }
        __syncthreads();
        const int bsel = sel_bucket;
        need -= sel_above;
        prefix |= static_cast<unsigned long long>(bsel) << sh;
        mask |= static_cast<unsigned long long>(dmask) << sh;
        const bool done = static_cast<int>(hist[bsel]) == need;
        __syncthreads();
        if (done || sh == 0) break;
    }

    // ---- ascending output: each thread owns a contiguous range of j; keys
    // above the bucket are kept, keys in it are kept lowest index first
    const int per = (T + STHREADS - 1) / STHREADS;
    const int jb = tid * per, je = min(T, jb + per);
    int n_eq = 0;
    for (int j = jb; j < je; ++j) n_eq += ((key_of(j) & mask) == prefix) ? 1 : 0;
    int tot;
    const int eq_rank = block_excl_scan(n_eq, scan_scratch, &tot);
    int n_sel = 0;
    {
        int r = eq_rank;
        for (int j = jb; j < je; ++j) {
            const unsigned long long km = key_of(j) & mask;
            if (km > prefix) ++n_sel;
            else if (km == prefix) n_sel += (r++ < need) ? 1 : 0;
        }
    }
    int pos = block_excl_scan(n_sel, scan_scratch, &tot);
    {
        int r = eq_rank;
        for (int j = jb; j < je; ++j) {
            const unsigned long long km = key_of(j) & mask;
            bool sel = km > prefix;
            if (km == prefix) sel = (r++ < need);
            if (sel) out[pos++] = j;
        }
    }
}

__global__ void iota_kernel(int32_t* __restrict__ idx, long long rows, int T) {
    const long long total = rows * T;
    for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x)
        idx[e] = static_cast<int32_t>(e % T);
}

inline size_t head_bytes(long long T) { return static_cast<size_t>(T) * static_cast<size_t>(T) * sizeof(double); }

}  // namespace topk
}  // namespace zb

using namespace zb;

extern "C" size_t zb_tile_score_topk_workspace_bytes(zb_shape s) {
    if (check_shape(s) != ZB_OK) return 0;
    const long long T = n_tiles(s);
    const int heads = s.heads < 4 ? s.heads : 4;  // up to 4 heads per pass by default
    return topk::head_bytes(T) * heads;
}

extern "C" zb_status zb_tile_score_topk(const double* Qbar, const double* Kbar, zb_shape s,
                                        int32_t k, int32_t* idx, void* ws, size_t ws_bytes,
                                        void* stream) {
    zb_status e = check_shape(s);
    if (e != ZB_OK) return e;
    if (!Qbar || !Kbar || (!idx && k > 0)) return ZB_ERR_NULL;
    const long long T = n_tiles(s);
    if (T > topk::MAX_T) return ZB_ERR_UNSUPPORTED;
    if (k < 0 || k > T) return ZB_ERR_SHAPE;
    if (!aligned16(Qbar) || !aligned16(Kbar) || !aligned16(idx) || !aligned16(ws)) return ZB_ERR_ALIGN;
    if (k == 0) return ZB_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (k == T) {  // keep-all: every row is 0..T-1, no scoring needed
        DeviceInfo dev;
        if ((e = current_device(&dev)) != ZB_OK) return e;
        topk::iota_kernel<<<4 * dev.sm_count, 256, 0, st>>>(idx, static_cast<long long>(s.heads) * T,
                                                            static_cast<int>(T));
        return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
    }
    if (!ws || ws_bytes < topk::head_bytes(T)) return ZB_ERR_WORKSPACE;
    DeviceInfo dev;
    if ((e = current_device(&dev)) != ZB_OK) return e;
    const size_t fit = ws_bytes / topk::head_bytes(T);
    const int per_pass = static_cast<int>(fit < static_cast<size_t>(s.heads) ? fit : static_cast<size_t>(s.heads));
    const size_t gsmem = 2 * topk::HD * topk::GS * sizeof(double);
    const size_t row_bytes = static_cast<size_t>(T) * sizeof(double);
    const int in_smem = row_bytes <= topk::SMEM_SCORE_LIMIT ? 1 : 0;
    const size_t ssmem = in_smem ? row_bytes : 0;
    if (cudaFuncSetAttribute(topk::score_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(gsmem)) != cudaSuccess ||
        cudaFuncSetAttribute(topk::select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(ssmem > 0 ? ssmem : 16)) != cudaSuccess)
        return ZB_ERR_CUDA;
    double* scores = static_cast<double*>(ws);
    const int blocks = static_cast<int>((T + topk::GT - 1) / topk::GT);
    for (int h0 = 0; h0 < s.heads; h0 += per_pass) {
        const int hn = (s.heads - h0) < per_pass ? (s.heads - h0) : per_pass;
        topk::score_gemm_kernel<<<dim3(blocks, blocks, hn), topk::GTHREADS, gsmem, st>>>(
            Qbar, Kbar, static_cast<int>(T), h0, scores);
        if (cudaGetLastError() != cudaSuccess) return ZB_ERR_CUDA;
        const long long rows = static_cast<long long>(hn) * T;
        if (rows > 0x7FFFFFFFll) return ZB_ERR_UNSUPPORTED;
        topk::select_kernel<<<static_cast<unsigned>(rows), topk::STHREADS, ssmem, st>>>(
            scores, static_cast<int>(T), k, h0, in_smem, idx);
        if (cudaGetLastError() != cudaSuccess) return ZB_ERR_CUDA;
    }
    return ZB_OK;
}
