// Closed-form affine fit of the linear stage to the dense output.
//
// "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D Reconstruction",
// Abstract: closed-form affine fitting makes the conversion training-free;
// Table 3 (a) compares the unfitted linear operator with fitted ones.  "Zebra3D
// speeds up 3D reconstruction by up to 7.1x on 1024 frames without training
// from scratch", section "How Zebra3D works": the fit needs no gradient
// descent.  Reading used: per head, least squares of [X 1] [A; b] = Y over the
// calibration rows (row vectors, y = x A + b).
//
// Solved in fp64 through centred normal equations (the intercept absorbs the
// means) with a vanishing ridge on A that keeps degenerate calibration sets
// solvable:
//   xm, ym = column means;  G = (X - xm)^T (X - xm);  C = (X - xm)^T (Y - ym);
//   lam = 1e-8 * max_i G_ii;  (G + lam I) A = C (Cholesky);  b = ym - xm A.
// Three kernels: column means per head; Gram partials per (head, 256-row
// chunk); fixed-order reduction + Cholesky + two triangular solves per head.
#include <cuda_runtime.h>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace aff {

constexpr int HD = 64;
constexpr int CHUNK = 256;
constexpr int BATCH = 32;  // rows staged in shared memory at a time
constexpr double RIDGE_REL = 1e-8;

inline long long n_chunks(long long rows) { return (rows + CHUNK - 1) / CHUNK; }

inline size_t ws_bytes(int heads, long long rows) {
    return static_cast<size_t>(heads) * (2 * HD + n_chunks(rows) * 2 * HD * HD) * sizeof(double);
}


// ws layout per head: [means: 2 x 64][partials: chunks x 2 x 64 x 64]
__global__ void __launch_bounds__(256) affine_means_kernel(const float* __restrict__ X, const float* __restrict__ Y,
                                    long long rows, double* __restrict__ ws, long long nch) {
    const int h = blockIdx.x;
    const int c = threadIdx.x & 63, r0 = threadIdx.x >> 6;
    __shared__ double red[2][4][HD];
    double sx = 0.0, sy = 0.0;
    const float* xh = X + static_cast<long long>(h) * rows * HD;
    const float* yh = Y + static_cast<long long>(h) * rows * HD;
    for (long long r = r0; r < rows; r += 4) {
        sx += static_cast<double>(xh[r * HD + c]);
        sy += static_cast<double>(yh[r * HD + c]);
    }
    red[0][r0][c] = sx;
    red[1][r0][c] = sy;
    __syncthreads();
    if (threadIdx.x < 2 * HD) {
        const int t = threadIdx.x >> 6, cc = threadIdx.x & 63;
        const double s = red[t][0][cc] + red[t][1][cc] + red[t][2][cc] + red[t][3][cc];
        ws[static_cast<size_t>(h) * (2 * HD + nch * 2 * HD * HD) + t * HD + cc] = s / static_cast<double>(rows);
    }
}

__global__ void __launch_bounds__(256) affine_gram_kernel(const float* __restrict__ X, const float* __restrict__ Y,
                                   long long rows, double* __restrict__ ws, long long nch) {
    const int h = blockIdx.y;
    const long long ch = blockIdx.x;
    __shared__ double xs[BATCH][HD], ys[BATCH][HD];
    __shared__ double mx[HD], my[HD];
    double* wh = ws + static_cast<size_t>(h) * (2 * HD + nch * 2 * HD * HD);
    if (threadIdx.x < HD) {
        mx[threadIdx.x] = wh[threadIdx.x];
        my[threadIdx.x] = wh[HD + threadIdx.x];
    }
    const int a = threadIdx.x >> 2;          // row of G / C
    const int b0 = (threadIdx.x & 3) * 16;   // 16 columns
    double g[16], cc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) g[e] = cc[e] = 0.0;
    const float* xh = X + static_cast<long long>(h) * rows * HD;
    const float* yh = Y + static_cast<long long>(h) * rows * HD;
    const long long rbeg = ch * CHUNK;
    const long long rend = min(rows, rbeg + CHUNK);
    __syncthreads();
    for (long long r0 = rbeg; r0 < rend; r0 += BATCH) {
        for (int e = threadIdx.x; e < BATCH * HD; e += blockDim.x) {
            const int rr = e / HD, col = e % HD;
            const long long r = r0 + rr;
            const bool in = r < rend;
            xs[rr][col] = in ? static_cast<double>(xh[r * HD + col]) - mx[col] : 0.0;
            ys[rr][col] = in ? static_cast<double>(yh[r * HD + col]) - my[col] : 0.0;
        }
        __syncthreads();
#pragma unroll 4
        for (int rr = 0; rr < BATCH; ++rr) {
            const double xa = xs[rr][a];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                g[e] = fma(xa, xs[rr][b0 + e], g[e]);
                cc[e] = fma(xa, ys[rr][b0 + e], cc[e]);
            }
        }
        __syncthreads();
    }
    double* part = wh + 2 * HD + ch * 2 * HD * HD;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        part[a * HD + b0 + e] = g[e];
        part[HD * HD + a * HD + b0 + e] = cc[e];
    }
}

__global__ void __launch_bounds__(HD) affine_solve_kernel(const double* __restrict__ ws, long long nch, float* __restrict__ A,
                                    float* __restrict__ bvec, int* status) {
    const int h = blockIdx.x;
    const int t = threadIdx.x;  // 64 threads
    extern __shared__ double dyn[];
    double (*G)[HD + 1] = reinterpret_cast<double (*)[HD + 1]>(dyn);
    double (*C)[HD + 1] = reinterpret_cast<double (*)[HD + 1]>(dyn + HD * (HD + 1));
    __shared__ int singular;
    const double* wh = ws + static_cast<size_t>(h) * (2 * HD + nch * 2 * HD * HD);
    // fixed-order sum of the chunk partials; thread t owns row t
    for (int j = 0; j < HD; ++j) {
        double sg = 0.0, sc = 0.0;
        for (long long c = 0; c < nch; ++c) {
            const double* p = wh + 2 * HD + c * 2 * HD * HD;
            sg += p[t * HD + j];
            sc += p[HD * HD + t * HD + j];
        }
        G[t][j] = sg;
        C[t][j] = sc;
    }
    if (t == 0) singular = 0;
    __syncthreads();
    // vanishing ridge: lam = RIDGE_REL * max_i G_ii (every thread computes it)
    {
        double gmax = 0.0;
        for (int i = 0; i < HD; ++i) gmax = fmax(gmax, G[i][i]);
        __syncthreads();
        G[t][t] += RIDGE_REL * gmax;
        __syncthreads();
    }
    // Cholesky G = L L^T in place (lower triangle), right-looking
    for (int j = 0; j < HD; ++j) {
        if (t == 0) {
            const double piv = G[j][j];
            if (!(piv > 0.0)) singular = 1;
            G[j][j] = sqrt(piv > 0.0 ? piv : 1.0);
        }
        __syncthreads();
        if (t > j) G[t][j] /= G[j][j];
        __syncthreads();
        if (t > j) {
            const double ltj = G[t][j];
            for (int k = j + 1; k <= t; ++k) G[t][k] = fma(-ltj, G[k][j], G[t][k]);
        }
        __syncthreads();
    }
    // thread t solves column t of A: L Y = C[:, t], then L^T X = Y
    for (int i = 0; i < HD; ++i) {
        double s = C[i][t];
        for (int k = 0; k < i; ++k) s = fma(-G[i][k], C[k][t], s);
        C[i][t] = s / G[i][i];
    }
    for (int i = HD - 1; i >= 0; --i) {
        double s = C[i][t];
        for (int k = i + 1; k < HD; ++k) s = fma(-G[k][i], C[k][t], s);
        C[i][t] = s / G[i][i];
    }
    __syncthreads();
    const bool bad = singular != 0;
    if (bad && t == 0) flag_status(status, ZB_ERR_SINGULAR);
    const double* mx = wh;
    const double* my = wh + HD;
    double bb = my[t];
    for (int i = 0; i < HD; ++i) bb = fma(-mx[i], C[i][t], bb);
    for (int i = 0; i < HD; ++i)
        A[static_cast<size_t>(h) * HD * HD + i * HD + t] = bad ? __int_as_float(0x7fc00000) : static_cast<float>(C[i][t]);
    bvec[static_cast<size_t>(h) * HD + t] = bad ? __int_as_float(0x7fc00000) : static_cast<float>(bb);
}

}  // namespace aff
}  // namespace zb

using namespace zb;

extern "C" size_t zb_affine_fit_workspace_bytes(int32_t heads, int64_t rows, int32_t head_dim) {
    if (heads < 1 || rows < 1 || head_dim != 64) return 0;
    return aff::ws_bytes(heads, rows);
}

extern "C" zb_status zb_affine_fit(const float* X, const float* Y, int32_t heads, int64_t rows,
                                   int32_t head_dim, float* A, float* b, void* ws, size_t ws_bytes,
                                   void* stream) {
    if (heads < 1) return ZB_ERR_SHAPE;
    if (head_dim != 64) return ZB_ERR_UNSUPPORTED;
    if (rows < head_dim + 1) return ZB_ERR_SHAPE;
    if (!X || !Y || !A || !b) return ZB_ERR_NULL;
    if (!aligned16(X) || !aligned16(Y) || !aligned16(A) || !aligned16(b) || !aligned16(ws)) return ZB_ERR_ALIGN;
    if (!ws || ws_bytes < aff::ws_bytes(heads, rows)) return ZB_ERR_WORKSPACE;
    const long long nch = aff::n_chunks(rows);
    if (nch > 65535) return ZB_ERR_UNSUPPORTED;
    DeviceInfo dev;
    zb_status e = current_device(&dev);
    if (e != ZB_OK) return e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    double* w = static_cast<double*>(ws);
    aff::affine_means_kernel<<<heads, 256, 0, st>>>(X, Y, rows, w, nch);
    if (cudaGetLastError() != cudaSuccess) return ZB_ERR_CUDA;
    aff::affine_gram_kernel<<<dim3(static_cast<unsigned>(nch), heads), 256, 0, st>>>(X, Y, rows, w, nch);
    if (cudaGetLastError() != cudaSuccess) return ZB_ERR_CUDA;
    const size_t smem = 2 * aff::HD * (aff::HD + 1) * sizeof(double);
    if (cudaFuncSetAttribute(aff::affine_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return ZB_ERR_CUDA;
    aff::affine_solve_kernel<<<heads, aff::HD, smem, st>>>(w, nch, A, b, dev.status);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}
