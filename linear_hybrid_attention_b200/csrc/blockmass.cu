// Block-mass diagnostic: the dense-softmax probability mass of every (query
// block, key block) pair, and the share of it that a selection keeps.
//
// "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D Reconstruction",
// Figure 2 (b) and Figure 8: the attention mass retained by the heaviest 20%
// of 64 x 64 token blocks, measured on a dense pass, shows how concentrated
// attention is in the sensitive stages.
//
// Two passes over K per query tile: zb_dense_attn gives every row's
// log-sum-exp; block_mass_kernel then recomputes S = Q K^T tile by tile on the
// tensor cores and sums p = exp(s q.k - lse) over 64- or 128-token blocks.
//   block_mass_kernel     one CTA of 4 warps per (query tile, head): thread 0
//                         issues the TMA loads (K in a ring of two) and the
//                         S MMA of the next key tile into the other of two
//                         TMEM buffers while all four warps turn the current
//                         S into block sums (one query row per thread);
//   top_mass_kernel       per row of M, the sum of its m largest entries over
//                         the row total (radix select on the float bits);
//   selected_mass_kernel  per row of M, the mass in the listed key tiles over
//                         the row total.
#include <cuda.h>
#include <cuda_runtime.h>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace bm {

constexpr int HD = 64;
constexpr int BM = 128;                          // query rows per CTA (MMA M)
constexpr int BN = 128;                          // keys per step (MMA N)
constexpr int THREADS = 128;                     // warp w reads TMEM lanes 32w..32w+31
constexpr uint32_t TILE_BYTES = BM * HD * 2;     // one 128 x 64 bf16 tile
constexpr uint32_t TMEM_COLS = 2 * BN;           // two fp32 S buffers
constexpr size_t SMEM_REQUEST = 96 * 1024;       // at most two CTAs per SM (TMEM: 2 x 256 columns)
constexpr float LOG2E = 1.4426950408889634f;
constexpr int MAX_BLOCKS = 49152;                // key blocks per row that top_mass_kernel holds in shared memory

struct __align__(1024) Smem {
    uint8_t q[TILE_BYTES];
    uint8_t k[2][TILE_BYTES];
    float red[2][THREADS / 32][2];  // per-warp sums of the last two key tiles (two key blocks each)
    uint64_t q_full, k_full[2], s_full[2], done;
    uint32_t tmem_base;
    int abort_flag;
};

// Writes the block masses of key tile jt from the per-warp sums in red[jt & 1]:
// block 64: rows 0..63 are warps 0, 1 and rows 64..127 warps 2, 3, columns
// 0..63 and 64..127 the two sums of a warp; block 128: all of it.  One thread
// per stored value, fixed order of the additions.
__device__ __forceinline__ void store_tile(const Smem& sm, int jt, int i, int h, int block, int Tb,
                                           float* __restrict__ M) {
    const int tid = threadIdx.x;
    const float(*r)[2] = sm.red[jt & 1];
    if (block == 64) {
        if (tid < 4) {
            const int qb = tid >> 1, kb = tid & 1;
            const int a = 2 * i + qb, b = 2 * jt + kb;
            if (a < Tb && b < Tb)
                M[(static_cast<long long>(h) * Tb + a) * Tb + b] = r[2 * qb][kb] + r[2 * qb + 1][kb];
        }
    } else if (tid == 0) {
        const float w0 = r[0][0] + r[0][1], w1 = r[1][0] + r[1][1];
        const float w2 = r[2][0] + r[2][1], w3 = r[3][0] + r[3][1];
        M[(static_cast<long long>(h) * Tb + i) * Tb + jt] = (w0 + w1) + (w2 + w3);
    }
}

__global__ void __launch_bounds__(THREADS, 2)
block_mass_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk, long long n,
                  int T, int block, int Tb, const float* __restrict__ lse, float scale_log2,
                  float* __restrict__ M, int* status, unsigned long long timeout_ns) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i = blockIdx.x, h = blockIdx.y;
    const WaitCtx wc{status, &sm.abort_flag, timeout_ns};

    if (tid == 0) {
        sm.abort_flag = 0;
        mbar_init(smem_addr(&sm.q_full), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&sm.k_full[s]), 1);
            mbar_init(smem_addr(&sm.s_full[s]), 1);
        }
        mbar_init(smem_addr(&sm.done), 1);
        fence_mbar_init();
        tma_prefetch_desc(&tq);
        tma_prefetch_desc(&tk);
    }
    if (warp == 0) tmem_alloc(smem_addr(&sm.tmem_base), TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    // this thread's query row and its normaliser in log2 units
    const long long qrow = static_cast<long long>(i) * BM + tid;
    const bool row_ok = qrow < n;
    const float l2 = row_ok ? __ldg(lse + static_cast<long long>(h) * n + qrow) * LOG2E : 0.f;

    int k_issued = 0;    // K tiles whose load thread 0 issued (in order)
    int k_consumed = 0;  // K tiles whose load thread 0 waited for
    bool q_waited = false;
    if (tid == 0) {
        mbar_arrive_expect_tx(smem_addr(&sm.q_full), TILE_BYTES);
        tma_load_3d(smem_addr(sm.q), &tq, smem_addr(&sm.q_full), 0, i * BM, h);
        for (int s = 0; s < 2 && s < T; ++s) {
            mbar_arrive_expect_tx(smem_addr(&sm.k_full[s]), TILE_BYTES);
            tma_load_3d(smem_addr(sm.k[s]), &tk, smem_addr(&sm.k_full[s]), 0, s * BN, h);
            ++k_issued;
        }
    }

    constexpr uint32_t IDESC = idesc_bf16(BM, BN, 0, 0);  // Q and K both K-major
    // S[j & 1] = Q K_j^T (thread 0); the buffer was read by every thread before
    // the block barrier that ended step j - 2
    auto issue_mma = [&](int j) -> bool {
        const int s = j & 1;
        if (!q_waited) {
            if (!mbar_wait(smem_addr(&sm.q_full), 0, wc)) return false;
            q_waited = true;
        }
        if (!mbar_wait(smem_addr(&sm.k_full[s]), (j >> 1) & 1, wc)) return false;
        ++k_consumed;
        tc_fence_after();
        const uint32_t qa = smem_addr(sm.q), ka = smem_addr(sm.k[s]);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
            umma_ss(tmem + s * BN, sdesc_sw128(qa + kk * 32, 16, 1024), sdesc_sw128(ka + kk * 32, 16, 1024), IDESC,
                    kk > 0 ? 1u : 0u);
        umma_commit(smem_addr(&sm.s_full[s]));
        return true;
    };

    bool ok = true;
    {
        bool good = true;
        if (tid == 0) good = issue_mma(0);
        if (__syncthreads_or(!good)) ok = false;
    }
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    for (int j = 0; ok && j < T; ++j) {
        const int s = j & 1;
        bool good = true;
        if (tid == 0 && j + 1 < T) good = issue_mma(j + 1);
        // the lanes of a warp agree before the warp-collective TMEM loads below
        // (lane 0 of warp 0 may have given up in issue_mma)
        good = __all_sync(0xffffffffu, good);
        if (good) good = mbar_wait_warp(smem_addr(&sm.s_full[s]), (j >> 1) & 1, wc);
        float sum0 = 0.f, sum1 = 0.f;
        if (good) {
            tc_fence_after();
            uint32_t raw[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) tmem_ld32(tmem + lane_addr + s * BN + c * 32, sub32(raw, c * 32));
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) tmem_wait_ld_dep(sub32(raw, c * 32));
            // MMA j has read K stage s: refill it with K_{j+2}
            if (tid == 0 && j + 2 < T) {
                mbar_arrive_expect_tx(smem_addr(&sm.k_full[s]), TILE_BYTES);
                tma_load_3d(smem_addr(sm.k[s]), &tk, smem_addr(&sm.k_full[s]), 0, (j + 2) * BN, h);
                ++k_issued;
            }
            // p = 2^(s q.k log2(e) - lse log2(e)); zero past the last key and for rows past n
            const long long keys_left = n - static_cast<long long>(j) * BN;
            const int valid = row_ok ? static_cast<int>(keys_left < BN ? keys_left : BN) : 0;
            const uint64_t c2 = f2_pack(scale_log2, scale_log2), nl2 = f2_pack(-l2, -l2);
            uint64_t acc[2][2] = {{0ull, 0ull}, {0ull, 0ull}};
#pragma unroll
            for (int e = 0; e < BN; e += 2) {
                float a0, a1;
                f2_unpack(f2_fma(f2_pack(__uint_as_float(raw[e]), __uint_as_float(raw[e + 1])), c2, nl2), a0, a1);
                const float p0 = e < valid ? ex2(a0) : 0.f;
                const float p1 = e + 1 < valid ? ex2(a1) : 0.f;
                uint64_t& dst = acc[e / 64][(e >> 1) & 1];
                dst = f2_add(dst, f2_pack(p0, p1));
            }
            float x0, x1, y0, y1;
            f2_unpack(f2_add(acc[0][0], acc[0][1]), x0, x1);
            f2_unpack(f2_add(acc[1][0], acc[1][1]), y0, y1);
            sum0 = x0 + x1;
            sum1 = y0 + y1;
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            sum0 += __shfl_xor_sync(0xffffffffu, sum0, o);
            sum1 += __shfl_xor_sync(0xffffffffu, sum1, o);
        }
        if (lane == 0) {
            sm.red[s][warp][0] = sum0;
            sm.red[s][warp][1] = sum1;
        }
        // the previous tile's sums were written before the barrier that ended step j - 1
        if (j > 0) store_tile(sm, j - 1, i, h, block, Tb, M);
        tc_fence_before();
        if (__syncthreads_or(!good)) {
            ok = false;
            break;
        }
    }
    if (ok) store_tile(sm, T - 1, i, h, block, Tb, M);

    // ---- drain: no MMA may run and no TMA may write once TMEM and shared memory go
    {
        volatile int no_abort = 0;
        const WaitCtx w2{status, &no_abort, drain_timeout_ns(timeout_ns)};
        if (tid == 0) {
            umma_commit(smem_addr(&sm.done));
            mbar_wait(smem_addr(&sm.done), 0, w2);
            if (!q_waited) mbar_wait(smem_addr(&sm.q_full), 0, w2);
            for (int q = k_consumed; q < k_issued; ++q) mbar_wait(smem_addr(&sm.k_full[q & 1]), (q >> 1) & 1, w2);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------ fractions ----
constexpr int SEL_THREADS = 256;

ZB_DEVINL double block_sum(double v, double* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
    if (threadIdx.x == 0) {
        for (int w = 0; w < SEL_THREADS / 32; ++w) t += red[w];
    }
    __syncthreads();
    return t;  // valid in thread 0
}

// One CTA per row of M [rows][Tb]: (sum of the row's m largest values) / (row
// sum).  Masses are >= 0, so their float bits order like their values; the
// m-th largest bit pattern is found digit by digit (4 passes of 8 bits).
__global__ void __launch_bounds__(SEL_THREADS)
top_mass_kernel(const float* __restrict__ M, int Tb, int m, float* __restrict__ frac) {
    extern __shared__ uint32_t keys[];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t s_prefix;
    __shared__ int s_want;
    __shared__ double red[SEL_THREADS / 32];
    const int tid = threadIdx.x;
    const long long row = blockIdx.x;
    const float* src = M + row * Tb;
    for (int t = tid; t < Tb; t += SEL_THREADS) {
        const float v = src[t];
        keys[t] = v > 0.f ? __float_as_uint(v) : 0u;
    }
    uint32_t prefix = 0, mask = 0;
    int want = m;  // rank (from the top, 1-based) still to find inside the current prefix
    for (int shift = 24; shift >= 0; shift -= 8) {
        hist[tid] = 0;  // SEL_THREADS == 256 bins
        __syncthreads();
        for (int t = tid; t < Tb; t += SEL_THREADS) {
            const uint32_t k = keys[t];
            if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid == 0) {
            int acc = 0, d = 255;
            for (; d > 0; --d) {
                if (acc + static_cast<int>(hist[d]) >= want) break;
                acc += static_cast<int>(hist[d]);
            }
            s_prefix = prefix | (static_cast<uint32_t>(d) << shift);
            s_want = want - acc;
        }
        __syncthreads();
        prefix = s_prefix;
        want = s_want;
        mask |= 255u << shift;
    }
    // prefix: bits of the m-th largest value v; take every value above v and `want` copies of v
    double top = 0.0, tot = 0.0;
    for (int t = tid; t < Tb; t += SEL_THREADS) {
        const uint32_t k = keys[t];
        const double v = static_cast<double>(__uint_as_float(k));
        tot += v;
        if (k > prefix) top += v;
    }
    top = block_sum(top, red);
    tot = block_sum(tot, red);
    if (tid == 0) {
        top += static_cast<double>(want) * static_cast<double>(__uint_as_float(prefix));
        frac[row] = tot > 0.0 ? static_cast<float>(top / tot) : 0.f;
    }
}

// One warp per row of M [rows][T]: (mass in the k listed key tiles) / (row sum).
__global__ void __launch_bounds__(SEL_THREADS)
selected_mass_kernel(const float* __restrict__ M, long long rows, int T, const int32_t* __restrict__ idx, int k,
                     float* __restrict__ frac, int* status) {
    const long long row = static_cast<long long>(blockIdx.x) * (SEL_THREADS / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;  // whole warps only
    const float* r = M + row * T;
    const int32_t* list = idx + row * k;
    double tot = 0.0, sel = 0.0;
    for (int t = lane; t < T; t += 32) tot += static_cast<double>(r[t]);
    bool bad = false;
    for (int q = lane; q < k; q += 32) {
        const int t = __ldg(list + q);
        if (t >= 0 && t < T) sel += static_cast<double>(r[t]);
        else bad = true;
    }
    if (bad) flag_status(status, ZB_ERR_INDEX);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        tot += __shfl_xor_sync(0xffffffffu, tot, o);
        sel += __shfl_xor_sync(0xffffffffu, sel, o);
    }
    if (lane == 0) frac[row] = tot > 0.0 ? static_cast<float>(sel / tot) : 0.f;
}

}  // namespace bm
}  // namespace zb

using namespace zb;

extern "C" zb_status zb_block_mass(const uint16_t* Q, const uint16_t* K, const float* lse, zb_shape s, float scale,
                                   float* M, void* stream) {
    zb_status e = check_shape(s);
    if (e != ZB_OK) return e;
    if (!Q || !K || !lse || !M) return ZB_ERR_NULL;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(M)) return ZB_ERR_ALIGN;
    if (!(scale > 0.f)) return ZB_ERR_SHAPE;
    if (s.heads > 65535) return ZB_ERR_UNSUPPORTED;
    const long long T = (s.n_tokens + bm::BM - 1) / bm::BM;
    const long long Tb = (s.n_tokens + s.tile - 1) / s.tile;
    if (T > 0x7FFFFFFFll || Tb > bm::MAX_BLOCKS) return ZB_ERR_UNSUPPORTED;
    DeviceInfo dev;
    if ((e = current_device(&dev)) != ZB_OK) return e;
    CUtensorMap mq, mk;
    if ((e = make_map_bf16_3d(&mq, Q, 64, s.n_tokens, s.heads, bm::BM)) != ZB_OK) return e;
    if ((e = make_map_bf16_3d(&mk, K, 64, s.n_tokens, s.heads, bm::BN)) != ZB_OK) return e;
    const size_t need = sizeof(bm::Smem) + 1024;
    const size_t smem = need > bm::SMEM_REQUEST ? need : bm::SMEM_REQUEST;
    if (cudaFuncSetAttribute(bm::block_mass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return ZB_ERR_CUDA;
    bm::block_mass_kernel<<<dim3(static_cast<unsigned>(T), static_cast<unsigned>(s.heads)), bm::THREADS, smem,
                            static_cast<cudaStream_t>(stream)>>>(mq, mk, s.n_tokens, static_cast<int>(T), s.tile,
                                                                 static_cast<int>(Tb), lse,
                                                                 scale * bm::LOG2E, M, dev.status, wait_timeout_ns());
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}

extern "C" zb_status zb_block_mass_top_fraction(const float* M, int32_t heads, int32_t n_blocks, int32_t m,
                                                float* frac, void* stream) {
    if (heads < 1 || n_blocks < 1 || m < 0 || m > n_blocks) return ZB_ERR_SHAPE;
    if (n_blocks > bm::MAX_BLOCKS) return ZB_ERR_UNSUPPORTED;
    if (!M || !frac) return ZB_ERR_NULL;
    if (!aligned16(M)) return ZB_ERR_ALIGN;
    const long long rows = static_cast<long long>(heads) * n_blocks;
    if (rows > 0x7FFFFFFFll) return ZB_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (m == 0) return cudaMemsetAsync(frac, 0, rows * sizeof(float), st) == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
    const size_t smem = static_cast<size_t>(n_blocks) * sizeof(uint32_t);
    if (cudaFuncSetAttribute(bm::top_mass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return ZB_ERR_CUDA;
    bm::top_mass_kernel<<<static_cast<unsigned>(rows), bm::SEL_THREADS, smem, st>>>(M, n_blocks, m, frac);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}

extern "C" zb_status zb_block_mass_selected_fraction(const float* M, int32_t heads, int32_t n_blocks,
                                                     const int32_t* idx, int32_t k, float* frac, void* stream) {
    if (heads < 1 || n_blocks < 1 || k < 1 || k > n_blocks) return ZB_ERR_SHAPE;
    if (!M || !idx || !frac) return ZB_ERR_NULL;
    if (!aligned16(M)) return ZB_ERR_ALIGN;
    DeviceInfo dev;
    zb_status e = current_device(&dev);
    if (e != ZB_OK) return e;
    const long long rows = static_cast<long long>(heads) * n_blocks;
    const long long blocks = (rows + bm::SEL_THREADS / 32 - 1) / (bm::SEL_THREADS / 32);
    if (blocks > 0x7FFFFFFFll) return ZB_ERR_UNSUPPORTED;
    bm::selected_mass_kernel<<<static_cast<unsigned>(blocks), bm::SEL_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
        M, rows, n_blocks, idx, k, frac, dev.status);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}
