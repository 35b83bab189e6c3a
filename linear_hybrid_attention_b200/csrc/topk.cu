// Tile selection: the k largest mean-pooled scores Qbar_i . Kbar_j per query
// tile, exactly as fp64 scores order them.
//
// "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D Reconstruction",
// Figure 1 (a) caption names "selected tiles"; the pages give no criterion.
// Reading used: score(i, j) = Qbar_i . Kbar_j in fp64, the k largest kept,
// equal scores resolved toward the lower key-tile index, output ascending.
//
// The scores are not computed in fp64 for every pair.  Instead:
//  * digits_kernel: each row of Qbar and Kbar (64 fp64 values) becomes a
//    21-bit fixed-point integer vector m = trunc(x 2^(21 - e)) with one
//    power-of-two exponent e per row (max |x| < 2^e), split into three signed
//    7-bit digit planes d0, d1, d2 (m = d0 2^14 + d1 2^7 + d2).
//  * head_info_kernel: per head the largest key-row exponent e_ref, and
//    whether any key row is not finite.
//  * score_i8_kernel: tcgen05.mma kind::i8 (exact int32 accumulation) of the
//    digit products of weight 2^28, 2^21 and 2^14 (the three lower-weight
//    products are dropped), combined per (i, j) into the approximate score
//      s~_ij = (2^14 acc0 + 2^7 acc1 + acc2) 2^(14 + e_j - e_ref)   (fp32),
//    which is sigma_ij = s_ij 2^(42 - e_i - e_ref) (a positive factor fixed per
//    query row) up to |sigma64_ij - s~_ij| <= E, E = 2^29 + 2^25, where
//    sigma64 is the same scaling of the fp64 dot product.  Terms: truncation
//    of both rows < 64 (2^22) = 2^28; dropped digit products <= 64 * 127^2 *
//    (2^7 + 2^7 + 1) < 2^28; fp32 rounding of the combination <= 2^10.1 times a
//    scale <= 2^14; the fp64 dot product's own error <= 64 u 2^48 < 4.
//  * select_kernel (one CTA of 256 threads per query row, four per SM): a
//    2,048-bin linear histogram of s~ over [min, max] brackets the k-th largest
//    s~ between L and U; key tiles with s~ > U + 2E are certainly kept, those
//    with s~ < L - 2E certainly dropped.  The few in the band between are
//    re-scored in fp64 (one warp per tile) and ranked by (score, index); the
//    band's top (k - #kept) join the kept set, which is written ascending.
//    With tau the k-th largest s~ (L <= tau <= U): a tile ranked above a kept
//    one has s~ > U, and at most k - 1 tiles do; each of the >= k tiles with
//    s~ >= tau ranks above a dropped one.  So the result is the fp64
//    selection whatever the band holds.  Rows whose band exceeds 128
//    entries (ties, constant rows) resolve it with a radix select over the
//    fp64 keys, re-scoring band tiles in every pass; rows of heads with a
//    non-finite value treat every tile as band.
#include <cuda_runtime.h>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace topk {

constexpr int HD = 64;
constexpr int MAX_T = 32768;
constexpr int S_BITS = 21;                  // fixed-point bits of a row's values
constexpr int EXP_ZERO = -(1 << 29);        // exponent tag of an all-zero row
constexpr int EXP_NONFINITE = 1 << 29;      // exponent tag of a row holding inf or NaN
constexpr int DREC = 3 * HD;                // bytes of one row's digit planes d0 | d1 | d2
constexpr double E_BOUND = 570425344.0;     // 2^29 + 2^25

// Order-preserving map of an fp64 value to uint64 (larger value -> larger key);
// -0.0 is folded onto +0.0 so that they tie.
__device__ __forceinline__ unsigned long long order_key(double s) {
    if (s == 0.0) s = 0.0;
    const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(s));
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// ----------------------------------------------------------- digits ----
// One warp per row; rows [0, hn T) are Qbar's rows of heads h0.., then Kbar's.
__global__ void __launch_bounds__(256)
digits_kernel(const double* __restrict__ Qbar, const double* __restrict__ Kbar, long long T, int h0, int hn,
              int8_t* __restrict__ qd, int8_t* __restrict__ kd, int* __restrict__ qe, int* __restrict__ ke) {
    const long long per = static_cast<long long>(hn) * T;
    const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (r >= 2 * per) return;
    const int lane = threadIdx.x & 31;
    const bool is_k = r >= per;
    const long long rr = is_k ? r - per : r;  // hl * T + tile
    const double* src = (is_k ? Kbar : Qbar) + (static_cast<long long>(h0) * T + rr) * HD;
    const double2 v = reinterpret_cast<const double2*>(src)[lane];
    const bool bad = __any_sync(0xffffffffu, !isfinite(v.x) || !isfinite(v.y));
    double m = fmax(fabs(v.x), fabs(v.y));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    int e = 0;
    if (bad) e = EXP_NONFINITE;
    else if (m == 0.0) e = EXP_ZERO;
    else frexp(m, &e);  // m = f 2^e, 0.5 <= f < 1: every |x| < 2^e
    uint32_t planes[3] = {0u, 0u, 0u};
    if (e != EXP_NONFINITE && e != EXP_ZERO) {
        const double xs[2] = {v.x, v.y};
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            // exact scaling; |mi| <= 2^21 - 1
            const int mi = static_cast<int>(__double2ll_rz(scalbn(xs[u], S_BITS - e)));
            const int a = mi < 0 ? -mi : mi;
            const int d[3] = {a >> 14, (a >> 7) & 127, a & 127};
#pragma unroll
            for (int p = 0; p < 3; ++p) {
                const int s = mi < 0 ? -d[p] : d[p];
                planes[p] |= (static_cast<uint32_t>(s) & 0xFFu) << (8 * u);
            }
        }
    }
    int8_t* dst = (is_k ? kd : qd) + rr * DREC;
#pragma unroll
    for (int p = 0; p < 3; ++p)
        reinterpret_cast<uint16_t*>(dst + p * HD)[lane] = static_cast<uint16_t>(planes[p]);
    if (lane == 0) (is_k ? ke : qe)[rr] = e;
}

// One CTA per head: e_ref = the largest key-row exponent (0 if none), and
// whether a key row holds a non-finite value.
constexpr int HI_THREADS = 1024;
__global__ void __launch_bounds__(HI_THREADS) head_info_kernel(const int* __restrict__ ke, int T, int2* __restrict__ hinfo) {
    __shared__ int smax[HI_THREADS / 32], sbad[HI_THREADS / 32];
    const int hl = blockIdx.x;
    const int* e_h = ke + static_cast<long long>(hl) * T;
    int emax = -(1 << 30), bad = 0;
    for (int j = threadIdx.x; j < T; j += HI_THREADS) {
        const int e = e_h[j];
        if (e == EXP_NONFINITE) bad = 1;
        else if (e != EXP_ZERO) emax = max(emax, e);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
        bad |= __shfl_xor_sync(0xffffffffu, bad, o);
    }
    if ((threadIdx.x & 31) == 0) { smax[threadIdx.x >> 5] = emax; sbad[threadIdx.x >> 5] = bad; }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < HI_THREADS / 32; ++w) { emax = max(emax, smax[w]); bad |= sbad[w]; }
        hinfo[hl] = make_int2(emax == -(1 << 30) ? 0 : emax, bad);
    }
}

// --------------------------------------------------------- int8 GEMM ----
// Persistent: CTA c takes a contiguous range of the (head, query block, key
// block) tiles, 128 x 128 scores each.  The query block's digits stay in
// shared memory while the key blocks stream through two buffers (cp.async,
// issued while the MMAs of the previous tile run).  Both operands are K-major
// with the 128-byte swizzle: region x holds d0 | d1 (128 bytes a row), region y
// holds d2 in its first 64 bytes.  Thread 0 issues 12 MMAs (K = 32 bytes each)
// into three int32 TMEM accumulators (columns 0, 128, 256); eight warps read
// them back (warp w: lanes 32 (w % 4).., columns 64 (w / 4)..), combine them
// into fp32 scores and store each 256-byte row piece with a bulk copy.
constexpr int GTILE = 128;
constexpr int GTHREADS = 256;
constexpr int STAGE_LD = 68;  // floats per staged row piece (64 + 4: conflict-free float4 stores)

struct GemmSmem {
    uint8_t qx[GTILE * 128];
    uint8_t qy[GTILE * 128];
    uint8_t kx[2][GTILE * 128];
    uint8_t ky[2][GTILE * 128];
    float stage[GTHREADS * STAGE_LD];
    float colscale[2][GTILE];
    unsigned long long mma_bar;
    uint32_t tmem_base;
    int abort_flag;
};
constexpr size_t GEMM_SMEM = sizeof(GemmSmem) + 1024;  // + alignment of the base to 1024 bytes

// Instruction descriptor of tcgen05.mma kind::i8: signed 8-bit A and B, int32
// D, both operands K-major, M = N = 128.
constexpr uint32_t IDESC_S8 = (2u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

ZB_DEVINL void mma_s8(uint32_t d_tmem, uint32_t a_saddr, uint32_t b_saddr, uint32_t accumulate) {
    const uint64_t ad = sdesc_sw128(a_saddr, 16, 1024), bd = sdesc_sw128(b_saddr, 16, 1024);
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(ad), "l"(bd), "r"(IDESC_S8), "r"(accumulate)
        : "memory");
}

ZB_DEVINL void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem)), "l"(gmem) : "memory");
}
ZB_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
ZB_DEVINL void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Contiguous shared -> global copy (both 16-byte aligned, size a multiple of 16).
ZB_DEVINL void bulk_store(void* gdst, uint32_t ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                     reinterpret_cast<uint64_t>(gdst)),
                 "r"(ssrc), "r"(bytes)
                 : "memory");
}

// Rows [r0, r0 + 128) of a digit array (DREC bytes a row) into the swizzled
// regions x (chunks 0-7) and y (chunks 8-11); rows past T are zero.
ZB_DEVINL void load_digits(uint8_t* x, uint8_t* y, const int8_t* src, int r0, int T) {
    for (int e = threadIdx.x; e < GTILE * 12; e += GTHREADS) {
        const int r = e / 12, c = e % 12;
        uint8_t* dst = (c < 8 ? x : y) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
        if (r0 + r < T) cp_async16(dst, src + static_cast<long long>(r0 + r) * DREC + c * 16);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
}

// int32 in (-2^22, 2^22) -> fp32, exactly (through the bits of 1.5 * 2^23 + v)
ZB_DEVINL float small_i2f(uint32_t v) {
    return __int_as_float(static_cast<int>(v) + 0x4B400000) - 12582912.0f;
}

__global__ void __launch_bounds__(GTHREADS, 1)
score_i8_kernel(const int8_t* __restrict__ qd, const int8_t* __restrict__ kd, const int* __restrict__ ke,
                const int2* __restrict__ hinfo, int T, int Tp, int hn, float* __restrict__ scores, int* status,
                unsigned long long timeout_ns) {
    extern __shared__ uint8_t smem_raw[];
    GemmSmem& sm = *reinterpret_cast<GemmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long Tb = (T + GTILE - 1) / GTILE;
    const long long total = hn * Tb * Tb;
    const long long t0 = total * blockIdx.x / gridDim.x, t1 = total * (blockIdx.x + 1) / gridDim.x;
    if (t0 >= t1) return;
    if (tid == 0) {
        mbar_init(smem_addr(&sm.mma_bar), 1);
        fence_mbar_init();
        sm.abort_flag = 0;
    }
    if (warp == 0) tmem_alloc(smem_addr(&sm.tmem_base), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const WaitCtx wc{status, reinterpret_cast<volatile int*>(&sm.abort_flag), timeout_ns};

    auto load_cols = [&](int buf, int hl, int jb) {
        if (tid < GTILE) {
            const int j = jb * GTILE + tid;
            float sc = 0.f;
            if (j < T) {
                const int e = ke[static_cast<long long>(hl) * T + j];
                if (e != EXP_ZERO && e != EXP_NONFINITE) {
                    const int x = 14 + e - hinfo[hl].x;  // <= 14
                    if (x >= -126) sc = __int_as_float((x + 127) << 23);
                }
            }
            sm.colscale[buf][tid] = sc;
        }
    };
    auto split = [&](long long t, int& hl, int& ib, int& jb) {
        hl = static_cast<int>(t / (Tb * Tb));
        const long long r = t % (Tb * Tb);
        ib = static_cast<int>(r / Tb);
        jb = static_cast<int>(r % Tb);
    };

    int hl, ib, jb;
    split(t0, hl, ib, jb);
    load_digits(sm.kx[0], sm.ky[0], kd + static_cast<long long>(hl) * T * DREC, jb * GTILE, T);
    load_cols(0, hl, jb);
    cp_async_commit();
    long long cur_a = -1;
    uint32_t phase = 0;
    bool mma_pending = false;
    const int lq = warp & 3, hf = warp >> 2;
    float* piece = sm.stage + tid * STAGE_LD;
    for (long long t = t0; t < t1; ++t) {
        const int buf = static_cast<int>((t - t0) & 1);
        split(t, hl, ib, jb);
        const long long a_id = static_cast<long long>(hl) * Tb + ib;
        if (a_id != cur_a) {
            load_digits(sm.qx, sm.qy, qd + static_cast<long long>(hl) * T * DREC, ib * GTILE, T);
            cp_async_commit();
            cur_a = a_id;
        }
        cp_async_wait_all();
        fence_proxy_async_smem();  // the MMAs read these tiles through the async proxy
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t qx = smem_addr(sm.qx), qy = smem_addr(sm.qy);
            const uint32_t kx = smem_addr(sm.kx[buf]), ky = smem_addr(sm.ky[buf]);
            const uint32_t a0 = tmem, a1 = tmem + 128, a2 = tmem + 256;
            // weight 2^28: d0 . d0
            mma_s8(a0, qx, kx, 0u);
            mma_s8(a0, qx + 32, kx + 32, 1u);
            // weight 2^21: d0 . d1 + d1 . d0
            mma_s8(a1, qx, kx + 64, 0u);
            mma_s8(a1, qx + 32, kx + 96, 1u);
            mma_s8(a1, qx + 64, kx, 1u);
            mma_s8(a1, qx + 96, kx + 32, 1u);
            // weight 2^14: d0 . d2 + d1 . d1 + d2 . d0
            mma_s8(a2, qx, ky, 0u);
            mma_s8(a2, qx + 32, ky + 32, 1u);
            mma_s8(a2, qx + 64, kx + 64, 1u);
            mma_s8(a2, qx + 96, kx + 96, 1u);
            mma_s8(a2, qy, kx, 1u);
            mma_s8(a2, qy + 32, kx + 32, 1u);
            umma_commit(smem_addr(&sm.mma_bar));
        }
        mma_pending = true;
        if (t + 1 < t1) {  // the other buffer was last read by the MMAs of tile t - 1, which are done
            int hn1, ib1, jb1;
            split(t + 1, hn1, ib1, jb1);
            load_digits(sm.kx[buf ^ 1], sm.ky[buf ^ 1], kd + static_cast<long long>(hn1) * T * DREC, jb1 * GTILE, T);
            load_cols(buf ^ 1, hn1, jb1);
            cp_async_commit();
        }
        const bool got = mbar_wait_warp(smem_addr(&sm.mma_bar), phase, wc);
        if (__syncthreads_or(!got)) break;
        phase ^= 1u;
        mma_pending = false;
        tc_fence_after();
        bulk_wait_group_read<0>();  // this thread's previous store has read its staged piece
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * lq) << 16);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int col0 = 64 * hf + 32 * c;
            uint32_t r0[32], r1[32], r2[32];
            tmem_ld32(lane_base + col0, r0);
            tmem_ld32(lane_base + 128 + col0, r1);
            tmem_ld32(lane_base + 256 + col0, r2);
            tmem_wait_ld_dep(r0);
            tmem_wait_ld_dep(r1);
            tmem_wait_ld_dep(r2);
            const float* sc = sm.colscale[buf] + col0;
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                float o[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float p = fmaf(small_i2f(r0[e + u]), 16384.f, fmaf(small_i2f(r1[e + u]), 128.f, small_i2f(r2[e + u])));
                    o[u] = p * sc[e + u];
                }
                *reinterpret_cast<float4*>(piece + 32 * c + e) = make_float4(o[0], o[1], o[2], o[3]);
            }
        }
        const int row = ib * GTILE + 32 * lq + lane;
        if (row < T) {
            fence_proxy_async_smem();  // the bulk copy reads the piece through the async proxy
            bulk_store(scores + (static_cast<long long>(hl) * T + row) * Tp + jb * GTILE + 64 * hf, smem_addr(piece),
                       64 * sizeof(float));
            bulk_commit_group();
        }
        tc_fence_before();
        __syncthreads();  // TMEM read out before the next tile's MMAs overwrite it
    }
    cp_async_wait_all();  // a prefetch still in flight after an aborted wait
    bulk_wait_group<0>();
    if (mma_pending && warp == 0) {  // an aborted wait: let the MMAs finish before TMEM is freed
        volatile int no_abort = 0;
        const WaitCtx w2{status, &no_abort, drain_timeout_ns(timeout_ns)};
        mbar_wait_warp(smem_addr(&sm.mma_bar), phase, w2);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------ select ----
constexpr int STHREADS = 256;
constexpr int SWARPS = STHREADS / 32;
constexpr int NBINS = 2048;
constexpr int BPT = NBINS / STHREADS;  // bins per thread in the bucket search
constexpr int BAND_CAP = 128;
constexpr int DIGIT = 11;              // radix digit of the fp64 keys in a wide band
static_assert((1 << DIGIT) <= NBINS, "a radix digit's buckets must fit the histogram");
static_assert(BPT * STHREADS == NBINS, "bins per thread");

// Block-wide exclusive prefix sum of one int per thread.
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
    for (int w = 0; w < SWARPS; ++w) {
        const int s = scratch[w];
        if (w < warp) wsum += s;
        tot += s;
    }
    __syncthreads();
    *total = tot;
    return wsum + x - v;
}

// Block-wide exclusive suffix sum (the sum over higher-numbered threads).
__device__ __forceinline__ int block_excl_suffix(int v, int* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
    }
    if (lane == 0) scratch[warp] = x;
    __syncthreads();
    int above = 0;
#pragma unroll
    for (int w = 0; w < SWARPS; ++w)
        if (w > warp) above += scratch[w];
    __syncthreads();
    return above + x - v;
}

// The bucket of hist (counted from the top) that holds the need-th largest
// element: writes its index and the count above it.
ZB_DEVINL void find_bucket(const unsigned int* hist, int need, int* scratch, int* bucket, int* above_out) {
    unsigned int c[BPT];
    int local = 0;
#pragma unroll
    for (int e = 0; e < BPT; ++e) local += static_cast<int>(c[e] = hist[BPT * threadIdx.x + e]);
    const int above = block_excl_suffix(local, scratch);
    if (above < need && above + local >= need) {
        int run = above;
#pragma unroll
        for (int e = BPT - 1; e >= 0; --e) {
            if (run + static_cast<int>(c[e]) >= need) {
                *bucket = BPT * threadIdx.x + e;
                *above_out = run;
                break;
            }
            run += static_cast<int>(c[e]);
        }
    }
}

// fp64 score of one (query row, key tile): one FMA chain over d in index order.
ZB_DEVINL double score64(const double* q, const double* __restrict__ krow) {
    const double2* k2 = reinterpret_cast<const double2*>(krow);
    double acc = 0.0;
#pragma unroll 8
    for (int c = 0; c < HD / 2; ++c) {
        const double2 v = __ldg(k2 + c);
        acc = fma(q[2 * c], v.x, acc);
        acc = fma(q[2 * c + 1], v.y, acc);
    }
    return acc;
}

ZB_DEVINL int lin_bin(float v, float a, float c) {
    const int rb = __float_as_int(fmaf(v, a, c));  // monotone in v; 2^23 + bin for bins in range
    return min(max(rb, 0x4B000000) - 0x4B000000, NBINS - 1);
}

// grid: heads in group x T query rows.
__global__ void __launch_bounds__(STHREADS, 4)
select_kernel(const float* __restrict__ scores, const double* __restrict__ Qbar, const double* __restrict__ Kbar,
              const int* __restrict__ qe, const int2* __restrict__ hinfo, int T, int Tp, int k, int h0,
              int32_t* __restrict__ idx) {
    extern __shared__ __align__(16) float xs[];  // the row's approximate scores; then the kept words
    __shared__ unsigned int hist[NBINS];
    __shared__ int band_j[BAND_CAP];
    __shared__ unsigned long long band_key[BAND_CAP];
    __shared__ double qrow[HD];
    __shared__ int wcnt[SWARPS], scratch[SWARPS];
    __shared__ float red_mn[SWARPS], red_mx[SWARPS];
    __shared__ int nband, sel_bucket, sel_above;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hl = blockIdx.x / T, i = blockIdx.x % T;
    const long long h = h0 + hl;
    const float* grow = scores + (static_cast<long long>(hl) * T + i) * Tp;
    const double* kh = Kbar + h * T * HD;
    const int T4 = (T + 3) >> 2;
    unsigned int* kept_words = reinterpret_cast<unsigned int*>(xs + 4 * T4);

    float mn = INFINITY, mx = -INFINITY;
    for (int q = tid; q < T4; q += STHREADS) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(grow) + q);
        reinterpret_cast<float4*>(xs)[q] = v;
        const float w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (4 * q + u < T) { mn = fminf(mn, w[u]); mx = fmaxf(mx, w[u]); }
    }
    if (tid < HD) qrow[tid] = Qbar[(h * T + i) * HD + tid];
    bool exact = hinfo[hl].y != 0 || qe[static_cast<long long>(hl) * T + i] == EXP_NONFINITE;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) { red_mn[warp] = mn; red_mx[warp] = mx; }
    if (tid == 0) { nband = 0; sel_bucket = 0; sel_above = 0; }
    for (int b = tid; b < NBINS; b += STHREADS) hist[b] = 0u;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < SWARPS; ++w) { mn = fminf(mn, red_mn[w]); mx = fmaxf(mx, red_mx[w]); }

    // ---- bracket of the k-th largest approximate score, widened by 2E
    float lo_f = -INFINITY, hi_f = INFINITY;
    if (!exact) {
        const double range = static_cast<double>(mx) - static_cast<double>(mn);
        float a = range > 0.0 ? static_cast<float>(NBINS / range) : 0.f;
        if (!(a < 1e30f)) a = 0.f;
        const float c = static_cast<float>(8388608.0 - static_cast<double>(mn) * a);
        for (int q = tid; q < T4; q += STHREADS) {
            const float4 v = reinterpret_cast<const float4*>(xs)[q];
            const float w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (4 * q + u < T) atomicAdd(&hist[lin_bin(w[u], a, c)], 1u);
        }
        __syncthreads();
        find_bucket(hist, k, scratch, &sel_bucket, &sel_above);
        __syncthreads();
        const int b = sel_bucket;
        // v in bucket b  =>  v a + c in [2^23 + b - 1/2, 2^23 + b + 1/2] (bins 0 and 4095 open-ended)
        double L = mn, U = mx;
        if (a > 0.f) {
            if (b > 0) L = fmax(L, (8388608.0 + b - 1.0 - static_cast<double>(c)) / static_cast<double>(a));
            if (b < NBINS - 1) U = fmin(U, (8388608.0 + b + 1.0 - static_cast<double>(c)) / static_cast<double>(a));
        }
        const double slack = (fabs(static_cast<double>(mn)) + fabs(static_cast<double>(mx))) * 0x1p-40;
        lo_f = __double2float_rd(L - slack - 2.0 * E_BOUND);
        hi_f = __double2float_ru(U + slack + 2.0 * E_BOUND);
    }

    // ---- classify: kept (> hi), band, dropped (< lo).  Warp w owns the 32-aligned
    // range [w seg, (w+1) seg) and records the kept set as ballot words.
    const int seg = ((T + SWARPS - 1) / SWARPS + 31) & ~31;
    const int wb = warp * seg, we = min(T, wb + seg);
    auto classify = [&]() -> int {  // the kept words and the band list; returns #kept
        int kept = 0;
        for (int j0 = wb; j0 < we; j0 += 32) {
            const int j = j0 + lane;
            bool is_kept = false, is_band = false;
            if (j < we) {
                const float v = xs[j];
                is_kept = v > hi_f;
                is_band = exact || (v >= lo_f && v <= hi_f);
            }
            const unsigned int word = __ballot_sync(0xffffffffu, is_kept);
            if (lane == 0) kept_words[j0 >> 5] = word;
            kept += __popc(word);
            if (is_band) {
                const int slot = atomicAdd(&nband, 1);
                if (slot < BAND_CAP) band_j[slot] = j;
            }
        }
        if (lane == 0) wcnt[warp] = kept;
        __syncthreads();
        int kept_all = 0;
#pragma unroll
        for (int w = 0; w < SWARPS; ++w) kept_all += wcnt[w];
        return kept_all;
    };
    int kept_all = classify();
    int nb = nband;
    // The bracket guarantees 1 <= k - #kept <= #band.  Should that ever fail for a row,
    // the row is classified again with every tile in the band: the exact fp64 path.
    if (!(k - kept_all >= 1 && k - kept_all <= nb)) {
        __syncthreads();  // every thread has read nband and wcnt
        if (tid == 0) nband = 0;
        __syncthreads();
        exact = true;
        lo_f = -INFINITY;
        hi_f = INFINITY;
        kept_all = classify();
        nb = nband;
    }
    const int need = k - kept_all;

    if (nb <= BAND_CAP) {
        // ---- narrow band: fp64 scores (one warp per tile: lane l takes d = 2l, 2l + 1,
        // then a butterfly sum that leaves the same value in every lane), ranked by
        // (score desc, index asc); the band's top `need` join the kept words
        for (int t = warp; t < nb; t += SWARPS) {
            const double2 kv = __ldg(reinterpret_cast<const double2*>(kh + static_cast<long long>(band_j[t]) * HD) + lane);
            double acc = fma(qrow[2 * lane], kv.x, qrow[2 * lane + 1] * kv.y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) band_key[t] = order_key(acc);
        }
        __syncthreads();
        for (int t = tid; t < nb; t += STHREADS) {
            const unsigned long long kt = band_key[t];
            const int jt = band_j[t];
            int rank = 0;
            for (int u = 0; u < nb; ++u) {
                const unsigned long long ku = band_key[u];
                rank += (ku > kt || (ku == kt && band_j[u] < jt)) ? 1 : 0;
            }
            if (rank < need) atomicOr(&kept_words[jt >> 5], 1u << (jt & 31));
        }
        __syncthreads();
    } else {
        // ---- wide band: radix select over the band's fp64 keys, re-scored each pass
        auto in_band = [&](int j) -> bool {
            const float v = xs[j];
            return exact || (v >= lo_f && v <= hi_f);
        };
        auto key_of = [&](int j) -> unsigned long long {
            return order_key(score64(qrow, kh + static_cast<long long>(j) * HD));
        };
        unsigned long long prefix = 0, mask = 0;
        int rem = need;
        for (int shift = 64 - DIGIT;; shift -= DIGIT) {
            const int sh = shift < 0 ? 0 : shift;
            const int width = shift < 0 ? shift + DIGIT : DIGIT;
            const unsigned int dmask = (1u << width) - 1u;
            for (int b = tid; b < NBINS; b += STHREADS) hist[b] = 0u;
            if (tid == 0) { sel_bucket = 0; sel_above = 0; }
            __syncthreads();
            for (int j = tid; j < T; j += STHREADS) {
                if (!in_band(j)) continue;
                const unsigned long long key = key_of(j);
                if ((key & mask) == prefix) atomicAdd(&hist[static_cast<unsigned int>(key >> sh) & dmask], 1u);
            }
            __syncthreads();
            find_bucket(hist, rem, scratch, &sel_bucket, &sel_above);
            __syncthreads();
            const int bsel = sel_bucket;
            rem -= sel_above;
            prefix |= static_cast<unsigned long long>(bsel) << sh;
            mask |= static_cast<unsigned long long>(dmask) << sh;
            const bool done = static_cast<int>(hist[bsel]) == rem;
            __syncthreads();
            if (done || sh == 0) break;
        }
        // kept band tiles, in ascending j per thread range: above the prefix all, equal
        // ones lowest index first
        const int per = (T + STHREADS - 1) / STHREADS;
        const int rb = min(T, tid * per), re = min(T, rb + per);
        int n_eq = 0;
        for (int j = rb; j < re; ++j)
            if (in_band(j) && (key_of(j) & mask) == prefix) ++n_eq;
        int tot;
        int r = block_excl_scan(n_eq, scratch, &tot);
        for (int j = rb; j < re; ++j) {
            if (!in_band(j)) continue;
            const unsigned long long km = key_of(j) & mask;
            if (km > prefix || (km == prefix && r++ < rem)) atomicOr(&kept_words[j >> 5], 1u << (j & 31));
        }
        __syncthreads();
    }

    // ---- ascending output from the kept words: thread t takes words [t wpt, (t+1) wpt)
    const int nwords = (T + 31) >> 5;
    const int wpt = (nwords + STHREADS - 1) / STHREADS;
    const int w0 = min(nwords, tid * wpt), w1 = min(nwords, w0 + wpt);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(kept_words[w]);
    int total;
    int pos = block_excl_scan(cnt, scratch, &total);
    int32_t* out = idx + (h * T + i) * static_cast<long long>(k);
    for (int w = w0; w < w1; ++w) {
        unsigned int bits = kept_words[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1u;
            if (pos < k) out[pos] = 32 * w + b;
            ++pos;
        }
    }
}

__global__ void iota_kernel(int32_t* __restrict__ idx, long long rows, int T) {
    const long long total = rows * T;
    for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x)
        idx[e] = static_cast<int32_t>(e % T);
}

// Workspace of a group of hn heads: digit planes and exponents of Qbar and
// Kbar, the per-head summary and the fp32 score rows (Tp = T rounded up to 128
// columns), each region starting on a 256-byte boundary.
inline size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
struct Layout {
    size_t qd, kd, qe, ke, hinfo, scores, total;
};
inline Layout layout(long long T, int hn) {
    const size_t rows = static_cast<size_t>(T) * hn;
    const size_t Tp = static_cast<size_t>((T + GTILE - 1) / GTILE) * GTILE;
    Layout l;
    l.qd = 0;
    l.kd = l.qd + al256(rows * DREC);
    l.qe = l.kd + al256(rows * DREC);
    l.ke = l.qe + al256(rows * sizeof(int));
    l.hinfo = l.ke + al256(rows * sizeof(int));
    l.scores = l.hinfo + al256(hn * sizeof(int2));
    l.total = l.scores + al256(rows * Tp * sizeof(float));
    return l;
}

}  // namespace topk
}  // namespace zb

using namespace zb;

extern "C" size_t zb_tile_score_topk_workspace_bytes(zb_shape s) {
    if (check_shape(s) != ZB_OK) return 0;
    const long long T = n_tiles(s);
    const int heads = s.heads < 4 ? s.heads : 4;  // up to 4 heads per pass by default
    return topk::layout(T, 1).total * heads;
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
    DeviceInfo dev;
    if (k == T) {  // keep-all: every row is 0..T-1, no scoring needed
        if ((e = current_device(&dev)) != ZB_OK) return e;
        topk::iota_kernel<<<4 * dev.sm_count, 256, 0, st>>>(idx, static_cast<long long>(s.heads) * T,
                                                            static_cast<int>(T));
        return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
    }
    const size_t one = topk::layout(T, 1).total;
    if (!ws || ws_bytes < one) return ZB_ERR_WORKSPACE;
    if ((e = current_device(&dev)) != ZB_OK) return e;
    int per_pass = static_cast<int>(ws_bytes / one < static_cast<size_t>(s.heads) ? ws_bytes / one : s.heads);
    const int Tp = static_cast<int>((T + topk::GTILE - 1) / topk::GTILE) * topk::GTILE;
    const size_t ssmem = static_cast<size_t>((T + 3) / 4) * 16 + static_cast<size_t>((T + 31) / 32) * 4;
    if (cudaFuncSetAttribute(topk::score_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(topk::GEMM_SMEM)) != cudaSuccess ||
        cudaFuncSetAttribute(topk::select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(ssmem)) != cudaSuccess)
        return ZB_ERR_CUDA;
    uint8_t* base = static_cast<uint8_t*>(ws);
    const long long Tb = (T + topk::GTILE - 1) / topk::GTILE;
    for (int h0 = 0; h0 < s.heads; h0 += per_pass) {
        const int hn = (s.heads - h0) < per_pass ? (s.heads - h0) : per_pass;
        const topk::Layout l = topk::layout(T, hn);
        int8_t* qd = reinterpret_cast<int8_t*>(base + l.qd);
        int8_t* kd = reinterpret_cast<int8_t*>(base + l.kd);
        int* qe = reinterpret_cast<int*>(base + l.qe);
        int* ke = reinterpret_cast<int*>(base + l.ke);
        int2* hinfo = reinterpret_cast<int2*>(base + l.hinfo);
        float* scores = reinterpret_cast<float*>(base + l.scores);
        const long long drows = 2ll * hn * T;
        topk::digits_kernel<<<static_cast<unsigned>((drows + 7) / 8), 256, 0, st>>>(Qbar, Kbar, T, h0, hn, qd, kd,
                                                                                    qe, ke);
        topk::head_info_kernel<<<hn, topk::HI_THREADS, 0, st>>>(ke, static_cast<int>(T), hinfo);
        const long long tiles = hn * Tb * Tb;
        const int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
        topk::score_i8_kernel<<<grid, topk::GTHREADS, topk::GEMM_SMEM, st>>>(
            qd, kd, ke, hinfo, static_cast<int>(T), Tp, hn, scores, dev.status, wait_timeout_ns());
        const long long rows = static_cast<long long>(hn) * T;
        if (rows > 0x7FFFFFFFll) return ZB_ERR_UNSUPPORTED;
        topk::select_kernel<<<static_cast<unsigned>(rows), topk::STHREADS, ssmem, st>>>(
            scores, Qbar, Kbar, qe, hinfo, static_cast<int>(T), Tp, k, h0, idx);
        if (cudaGetLastError() != cudaSuccess) return ZB_ERR_CUDA;
    }
    return ZB_OK;
}
