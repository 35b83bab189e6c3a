// Linear attention (elu+1 feature map) with the per-head affine correction.
//
// "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D Reconstruction",
// Abstract: tolerant stages use linear attention; a closed-form affine fit
// makes the conversion training-free.  "Zebra3D speeds up 3D reconstruction by
// up to 7.1x on 1024 frames without training from scratch", section "How
// Zebra3D works": the linear parts are corrected by an affine map fitted in
// closed form.  Reading used (the pages give no formula): non-causal linear
// attention with phi(x) = elu(x) + 1 on unscaled q, k:
//   S = sum_r phi(k_r)^T v_r,  z = sum_r phi(k_r),
//   O_r = (phi(q_r) S / (phi(q_r) . z)) A + b.
//
// Both passes stream HBM once and put the d x d products on tcgen05:
//  * state: one CTA per (head pair, token chunk).  A 128-token step loads K
//    and V of two heads by TMA, applies phi to K in place (shared memory, same
//    swizzled layout; fp32 arithmetic on packed pairs, rounded to bf16) while
//    summing z, and issues
//        D[128 x 128] += [phi(K_h0)^T ; phi(K_h1)^T] . [V_h0 | V_h1]
//    (both operands MN-major); the diagonal 64 x 64 blocks are S_h0, S_h1.
//    Per-CTA partials are added in a fixed order by a second kernel.
//  * apply: persistent warp-specialised CTAs over (head, 128-token tile):
//    B = [ ((S - z c^T) A)^T ; z ; 0 ] (80 x 64, bf16) is built in shared
//    memory once per head, phi(Q) is applied in place in packed bf16, each
//    tile computes D[128 x 80] = phi(Q) B^T on the tensor core, and the
//    epilogue forms D[:, :64] / D[:, 64] + (c A + b) into a staging tile that
//    is stored with TMA.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace lin {

constexpr int HD = 64;
constexpr int TILE = 128;
constexpr uint32_t TILE_BYTES = TILE * HD * 2;  // 16 KB
constexpr int TARGET_CTAS = 148;                // one wave on a B200

// ------------------------------------------------------------ geometry ----
struct StateGeom {
    int pairs, chunks, tiles_per_chunk, n_tiles;
};

inline StateGeom state_geom(int heads, long long n) {
    StateGeom g;
    g.n_tiles = static_cast<int>((n + TILE - 1) / TILE);
    g.pairs = (heads + 1) / 2;
    int chunks = TARGET_CTAS / g.pairs;
    if (chunks < 1) chunks = 1;
    if (chunks > g.n_tiles) chunks = g.n_tiles;
    g.tiles_per_chunk = (g.n_tiles + chunks - 1) / chunks;
    g.chunks = (g.n_tiles + g.tiles_per_chunk - 1) / g.tiles_per_chunk;
    return g;
}

constexpr size_t PARTIAL_FLOATS = 2 * (HD * HD + HD);  // per CTA: S and z of two heads

inline size_t state_ws_bytes(int heads, long long n) {
    const StateGeom g = state_geom(heads, n);
    return static_cast<size_t>(g.pairs) * g.chunks * PARTIAL_FLOATS * sizeof(float);
}

ZB_DEVINL void named_bar_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// phi on a bf16 pair, in bf16 arithmetic (the result feeds a bf16 MMA operand):
// max(x, 0) + 2^(min(x, 0) * log2(e)).  log2(e) rounded to bf16 (1.4453125)
// perturbs e^x by a relative |x| * 1.8e-3, below the bf16 rounding of the
// result for |x| < 2 and on outputs that are small for larger |x|.
ZB_DEVINL uint32_t phi_bf16x2(uint32_t w) {
    constexpr uint32_t kLog2eBf16x2 = 0x3FB93FB9u;
    uint32_t pos, neg, e, r;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(pos) : "r"(w), "r"(0u));
    asm("min.bf16x2 %0, %1, %2;" : "=r"(neg) : "r"(w), "r"(0u));
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(neg) : "r"(neg), "r"(kLog2eBf16x2));
    asm("ex2.approx.ftz.bf16x2 %0, %1;" : "=r"(e) : "r"(neg));
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(pos), "r"(e));
    return r;
}

// phi(x) = elu(x) + 1 = max(x, 0) + exp(min(x, 0))  (x + 1 for x > 0, e^x otherwise)
__device__ __forceinline__ float phi(float x) {
    return fmaxf(x, 0.f) + ex2(fminf(x, 0.f) * 1.4426950408889634f);
}

// ============================================================== state ====
constexpr int ST_STAGES = 3;
constexpr int ST_THREADS = 512;  // 16 warps share the phi pass; warps 0..3 read TMEM

struct StateSmem {
    uint8_t buf[ST_STAGES][4][TILE_BYTES];  // [stage][K0, K1, V0, V1]
    float zred[ST_THREADS / 32][2][HD];
    uint64_t full[ST_STAGES], empty[ST_STAGES], done;
    uint32_t tmem_base;
    int abort_flag;
};

// Body of the state kernel.  CENTERED subtracts key_shift[h] (the head's mean
// key, fp32 [H][d]) from every key before phi: the linear-centered variant.
template <bool CENTERED>
__device__ __forceinline__ void linear_state_body(const CUtensorMap& tm_k, const CUtensorMap& tm_v, int heads,
                                                  long long n, StateGeom geo, float* __restrict__ partial,
                                                  int* status, unsigned long long timeout_ns,
                                                  const float* __restrict__ key_shift) {
    extern __shared__ uint8_t smem_raw[];
    StateSmem& sm = *reinterpret_cast<StateSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int pair = blockIdx.x / geo.chunks;
    const int chunk = blockIdx.x % geo.chunks;
    const int h0 = 2 * pair;
    const int h1 = min(2 * pair + 1, heads - 1);
    const int t_begin = chunk * geo.tiles_per_chunk;
    const int t_end = min(geo.n_tiles, t_begin + geo.tiles_per_chunk);
    const int steps = t_end - t_begin;
    const WaitCtx wc{status, &sm.abort_flag, timeout_ns};

    if (tid == 0) {
        sm.abort_flag = 0;
        for (int s = 0; s < ST_STAGES; ++s) {
            mbar_init(smem_addr(&sm.full[s]), 1);
            mbar_init(smem_addr(&sm.empty[s]), 1);
        }
        mbar_init(smem_addr(&sm.done), 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 0) tmem_alloc(smem_addr(&sm.tmem_base), 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    auto issue_load = [&](int step) {
        const int s = step % ST_STAGES;
        const uint32_t bar = smem_addr(&sm.full[s]);
        const int row = (t_begin + step) * TILE;
        mbar_arrive_expect_tx(bar, 4 * TILE_BYTES);
        tma_load_3d(smem_addr(sm.buf[s][0]), &tm_k, bar, 0, row, h0);
        tma_load_3d(smem_addr(sm.buf[s][1]), &tm_k, bar, 0, row, h1);
        tma_load_3d(smem_addr(sm.buf[s][2]), &tm_v, bar, 0, row, h0);
        tma_load_3d(smem_addr(sm.buf[s][3]), &tm_v, bar, 0, row, h1);
    };
    uint32_t issued = 0;  // loads issued by thread 0
    if (tid == 0) {
        for (int st = 0; st < ST_STAGES - 1 && st < steps; ++st) issue_load(st), ++issued;
    }

    constexpr uint32_t IDESC = idesc_bf16(128, 128, 1, 1);
    const int cg = tid & 7;        // logical 16-byte feature group
    const int rbase = tid >> 3;    // rows rbase + 64 m
    float z0[8], z1[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) z0[e] = z1[e] = 0.f;
    // the shifts of this thread's 8 features in both heads, as fp32 pairs
    uint64_t mu2[2][4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        mu2[0][e] = CENTERED ? f2_pack(__ldg(key_shift + h0 * HD + cg * 8 + 2 * e), __ldg(key_shift + h0 * HD + cg * 8 + 2 * e + 1))
                             : f2_pack(0.f, 0.f);
        mu2[1][e] = CENTERED ? f2_pack(__ldg(key_shift + h1 * HD + cg * 8 + 2 * e), __ldg(key_shift + h1 * HD + cg * 8 + 2 * e + 1))
                             : f2_pack(0.f, 0.f);
    }
    const uint64_t log2e2 = f2_pack(1.4426950408889634f, 1.4426950408889634f);
    bool ok = true;
    int consumed = 0;  // loads whose full barrier was waited on

    for (int st = 0; st < steps; ++st) {
        const int s = st % ST_STAGES;
        // a failed wait is not a break: every thread must reach the block barrier
        bool good = mbar_wait(smem_addr(&sm.full[s]), (st / ST_STAGES) & 1, wc);
        if (good) {
            consumed = st + 1;
            const long long row0 = static_cast<long long>(t_begin + st) * TILE;
            // phi(K) in place for both heads; rows past n become 0 (no contribution)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint8_t* kt = sm.buf[s][hh];
#pragma unroll
                for (int m = 0; m < TILE / (ST_THREADS / 8); ++m) {
                    const int r = rbase + (ST_THREADS / 8) * m;
                    uint4* p = reinterpret_cast<uint4*>(kt + r * 128 + ((cg ^ (r & 7)) << 4));
                    const uint4 v = *p;
                    uint32_t w[4] = {v.x, v.y, v.z, v.w};
                    const bool valid = row0 + r < n;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        uint64_t x2 = f2_pack(bf16_lo(w[e]), bf16_hi(w[e]));
                        if constexpr (CENTERED) x2 = f2_sub(x2, mu2[hh][e]);
                        float xa, xb;
                        f2_unpack(x2, xa, xb);
                        // phi(x) = max(x, 0) + 2^(min(x, 0) log2 e), where x - max(x, 0)
                        // is min(x, 0) exactly
                        const uint64_t pos = f2_pack(fmaxf(xa, 0.f), fmaxf(xb, 0.f));
                        float na, nb, a, b;
                        f2_unpack(f2_mul(f2_sub(x2, pos), log2e2), na, nb);
                        f2_unpack(f2_add(pos, f2_pack(ex2(na), ex2(nb))), a, b);
                        w[e] = valid ? pack_bf16x2(a, b) : 0u;
                        // z sums the bf16-rounded features that the MMA uses
                        if (hh == 0) { z0[2 * e] += bf16_lo(w[e]); z0[2 * e + 1] += bf16_hi(w[e]); }
                        else { z1[2 * e] += bf16_lo(w[e]); z1[2 * e + 1] += bf16_hi(w[e]); }
                    }
                    *p = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
        fence_proxy_async_smem();
        if (__syncthreads_or(!good)) { ok = false; break; }
        if (tid == 0) {
            tc_fence_after();
            const uint32_t a0 = smem_addr(sm.buf[s][0]);
            const uint32_t b0 = smem_addr(sm.buf[s][2]);
#pragma unroll
            for (int kk = 0; kk < TILE / 16; ++kk) {
                const uint64_t ad = sdesc_sw128(a0 + kk * 2048, TILE_BYTES, 1024);
                const uint64_t bd = sdesc_sw128(b0 + kk * 2048, TILE_BYTES, 1024);
                umma_ss(tmem, ad, bd, IDESC, (st > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(smem_addr(&sm.empty[s]));
            // refill the stage used by the previous step once its MMA is done;
            // a failed wait surfaces at the next block barrier via the abort flag
            const int nxt = st + ST_STAGES - 1;
            if (nxt < steps) {
                const int ps = nxt % ST_STAGES;
                bool free_ok = true;
                if (nxt >= ST_STAGES)
                    free_ok = mbar_wait(smem_addr(&sm.empty[ps]), ((nxt / ST_STAGES) - 1) & 1, wc);
                if (free_ok) issue_load(nxt), ++issued;
            }
        }
    }

    // ---- drain: no MMA may run and no TMA may write once we read and free
    {
        volatile int no_abort = 0;
        const WaitCtx w2{status, &no_abort, drain_timeout_ns(timeout_ns)};
        if (tid == 0) {
            umma_commit(smem_addr(&sm.done));
            for (uint32_t q = static_cast<uint32_t>(consumed); q < issued; ++q)
                mbar_wait(smem_addr(&sm.full[q % ST_STAGES]), (q / ST_STAGES) & 1, w2);
        }
        if (!mbar_wait(smem_addr(&sm.done), 0, w2)) ok = false;
        if (sm.abort_flag) ok = false;
    }
    tc_fence_after();
    float* part = partial + static_cast<size_t>(blockIdx.x) * PARTIAL_FLOATS;
    if (steps > 0 && ok && tid < 128) {
        const int hs = tid >> 6;   // head slot of this TMEM lane
        const int f = tid & 63;    // feature row
        uint32_t r[64];
        const uint32_t ta = tmem + (static_cast<uint32_t>(warp * 32) << 16) + hs * 64;
        tmem_ld32(ta, sub32(r, 0));
        tmem_ld32(ta + 32, sub32(r, 32));
        tmem_wait_ld_dep(sub32(r, 0));
        tmem_wait_ld_dep(sub32(r, 32));
        float4* dst = reinterpret_cast<float4*>(part + hs * (HD * HD) + f * HD);
#pragma unroll
        for (int c = 0; c < 16; ++c)
            dst[c] = make_float4(__uint_as_float(r[4 * c]), __uint_as_float(r[4 * c + 1]),
                                 __uint_as_float(r[4 * c + 2]), __uint_as_float(r[4 * c + 3]));
    } else if (!(steps > 0 && ok)) {
        for (int e = tid; e < 2 * HD * HD; e += ST_THREADS) part[e] = 0.f;
    }
    // z: lanes cg, cg+8, cg+16, cg+24 of a warp share a feature group
#pragma unroll
    for (int e = 0; e < 8; ++e) {
#pragma unroll
        for (int o = 8; o <= 16; o <<= 1) {
            z0[e] += __shfl_xor_sync(0xffffffffu, z0[e], o);
            z1[e] += __shfl_xor_sync(0xffffffffu, z1[e], o);
        }
    }
    if (lane < 8) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sm.zred[warp][0][cg * 8 + e] = z0[e];
            sm.zred[warp][1][cg * 8 + e] = z1[e];
        }
    }
    __syncthreads();
    if (tid < 128) {
        const int hs = tid >> 6, f = tid & 63;
        float zz = 0.f;
#pragma unroll
        for (int w = 0; w < ST_THREADS / 32; ++w) zz += sm.zred[w][hs][f];
        part[2 * HD * HD + hs * HD + f] = (steps > 0 && ok) ? zz : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

__global__ void __launch_bounds__(ST_THREADS, 1)
linear_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    int heads, long long n, StateGeom geo, float* __restrict__ partial, int* status,
                    unsigned long long timeout_ns) {
    linear_state_body<false>(tm_k, tm_v, heads, n, geo, partial, status, timeout_ns, nullptr);
}

__global__ void __launch_bounds__(ST_THREADS, 1)
linear_state_centered_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                             int heads, long long n, StateGeom geo, float* __restrict__ partial, int* status,
                             unsigned long long timeout_ns, const float* __restrict__ key_shift) {
    linear_state_body<true>(tm_k, tm_v, heads, n, geo, partial, status, timeout_ns, key_shift);
}

// Fixed-order sum of the per-CTA partials: S[h], z[h].
__global__ void linear_state_reduce_kernel(const float* __restrict__ partial, int heads, StateGeom geo,
                                           float* __restrict__ S, float* __restrict__ z) {
    const int h = blockIdx.x;
    const int pair = h >> 1, slot = h & 1;
    for (int e = threadIdx.x; e < HD * HD + HD; e += blockDim.x) {
        const size_t off = e < HD * HD ? static_cast<size_t>(slot) * HD * HD + e
                                       : 2 * HD * HD + static_cast<size_t>(slot) * HD + (e - HD * HD);
        float acc = 0.f;
        for (int c = 0; c < geo.chunks; ++c)
            acc += partial[static_cast<size_t>(pair * geo.chunks + c) * PARTIAL_FLOATS + off];
        if (e < HD * HD) S[static_cast<size_t>(h) * HD * HD + e] = acc;
        else z[static_cast<size_t>(h) * HD + (e - HD * HD)] = acc;
    }
}

// =========================================================== key mean ====
// Per-head mean key mu_h = (1/N) sum_r k_r, the shift of the linear-centered
// variant.  HBM stream over K: grid (chunks, heads); a CTA owns a contiguous
// run of rows of one head, thread t reads the 16-byte feature group t % 8 of
// rows t / 8, t / 8 + 32, ... (consecutive threads read consecutive 16 bytes),
// four rows in flight per thread, and sums them in fp32.  The 32 row lanes of
// a feature group are added in fp64 in a fixed order, the chunks likewise in
// a second kernel, so the result does not depend on scheduling.
constexpr int KM_THREADS = 256;
constexpr int KM_ROW_LANES = KM_THREADS / 8;  // rows per pass
constexpr int KM_UNROLL = 4;
constexpr int KM_TARGET_CTAS = 148 * 8;       // eight 256-thread CTAs per SM

inline int key_mean_chunks(int heads, long long n) {
    long long c = (KM_TARGET_CTAS + heads - 1) / heads;
    const long long max_c = (n + KM_ROW_LANES * KM_UNROLL - 1) / (KM_ROW_LANES * KM_UNROLL);
    if (c > max_c) c = max_c;
    if (c < 1) c = 1;
    return static_cast<int>(c);
}

ZB_DEVINL void add8_f32(float (&acc)[8], const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc[2 * e] += bf16_lo(w[e]);
        acc[2 * e + 1] += bf16_hi(w[e]);
    }
}

__global__ void __launch_bounds__(KM_THREADS)
key_sum_kernel(const uint16_t* __restrict__ K, long long n, int chunks, double* __restrict__ partial) {
    __shared__ double red[KM_THREADS / 32][HD];
    const int h = blockIdx.y, c = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cg = tid & 7, rl = tid >> 3;
    const long long per = (n + chunks - 1) / chunks;
    const long long r0 = static_cast<long long>(c) * per;
    const long long r1 = min(n, r0 + per);
    const uint4* rows = reinterpret_cast<const uint4*>(K + static_cast<long long>(h) * n * HD);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    long long r = r0 + rl;
    for (; r + KM_ROW_LANES * (KM_UNROLL - 1) < r1; r += KM_ROW_LANES * KM_UNROLL) {
        uint4 v[KM_UNROLL];
#pragma unroll
        for (int u = 0; u < KM_UNROLL; ++u) v[u] = __ldcs(rows + (r + KM_ROW_LANES * u) * 8 + cg);
#pragma unroll
        for (int u = 0; u < KM_UNROLL; ++u) add8_f32(acc, v[u]);
    }
    for (; r < r1; r += KM_ROW_LANES) add8_f32(acc, __ldcs(rows + r * 8 + cg));
    // lanes l, l ^ 8, l ^ 16, l ^ 24 of a warp hold the same feature group
    double dacc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        dacc[e] = static_cast<double>(acc[e]);
        dacc[e] += __shfl_xor_sync(0xffffffffu, dacc[e], 8);
        dacc[e] += __shfl_xor_sync(0xffffffffu, dacc[e], 16);
    }
    if (lane < 8) {
#pragma unroll
        for (int e = 0; e < 8; ++e) red[warp][cg * 8 + e] = dacc[e];
    }
    __syncthreads();
    if (tid < HD) {
        double sum = 0.0;
#pragma unroll
        for (int w = 0; w < KM_THREADS / 32; ++w) sum += red[w][tid];
        partial[(static_cast<long long>(h) * chunks + c) * HD + tid] = sum;
    }
}

__global__ void key_mean_reduce_kernel(const double* __restrict__ partial, int chunks, long long n,
                                       float* __restrict__ mu) {
    const int h = blockIdx.x, f = threadIdx.x;
    double sum = 0.0;
    for (int c = 0; c < chunks; ++c) sum += partial[(static_cast<long long>(h) * chunks + c) * HD + f];
    mu[h * HD + f] = static_cast<float>(sum / static_cast<double>(n));
}

// ============================================================== apply ====
// Warp-specialised, one persistent CTA per SM, each with a contiguous range of
// (head, 128-row tile) items:
//   warp 0       TMA producer of the Q tiles (ring of AP_STAGES);
//   warp 1       MMA issuer: D[128 x 80] = phi(Q) B^T into one of D_BUFS TMEM
//                accumulators (80 of 128 columns each);
//   warps 2..5   phi in place on each Q tile in shared memory, and the B
//                operand / bias of each new head;
//   warps 6..13  epilogue, two warps per TMEM lane quarter (warp w reads lanes
//                32 (w % 4).., columns 32 ((w - 6) / 4)..): O = D / D[64] + b'
//                for half a row per thread, into a swizzled staging tile.
// The roles only meet at mbarriers, so loads, phi, MMA and stores of
// successive tiles overlap.
constexpr int AP_STAGES = 6;
constexpr int AP_THREADS = 448;
constexpr int D_BUFS = 4;
constexpr int BN_ROWS = 80;  // 64 columns of S A, one of z, 15 of zeros
constexpr uint32_t B_BYTES = BN_ROWS * 128;
constexpr int PHI_BAR = 1;   // named barrier of the operand builders (warps 2..5, 128 threads)
constexpr int PHI_THREADS = 128;  // warps 2..5 apply phi
constexpr int EPI_BAR = 2;        // named barrier of the epilogue warps (256 threads)
constexpr int EPI_THREADS = 256;

struct ApplySmem {
    uint8_t q[AP_STAGES][TILE_BYTES];
    uint8_t ost[2][TILE_BYTES];   // output tiles (128-byte swizzle) for the TMA store
    uint8_t bop[2][B_BYTES];
    float bvec[2][HD];
    float cvec[HD];
    uint64_t q_full[AP_STAGES], q_empty[AP_STAGES], phi_done[AP_STAGES];
    uint64_t mma_done[D_BUFS], d_free[D_BUFS];
    uint64_t b_free[2];       // MMAs of the last head that used bop / bvec [i] are done
    uint64_t bvec_ready[2];   // bvec [i] written for its head
    uint64_t bvec_free[2];    // the epilogue is past the last head that read bvec [i]
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

__global__ void __launch_bounds__(AP_THREADS, 1)
linear_apply_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
                    int heads, long long n_q, const float* __restrict__ S, const float* __restrict__ z,
                    const float* __restrict__ A, const float* __restrict__ bias, int* status,
                    unsigned long long timeout_ns) {
    extern __shared__ uint8_t smem_raw[];
    ApplySmem& sm = *reinterpret_cast<ApplySmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Tn = static_cast<int>((n_q + TILE - 1) / TILE);
    const long long n_items = static_cast<long long>(heads) * Tn;
    const long long per = (n_items + gridDim.x - 1) / gridDim.x;
    const long long first = static_cast<long long>(blockIdx.x) * per;
    const long long last = min(n_items, first + per);
    const int cnt = first < last ? static_cast<int>(last - first) : 0;
    const WaitCtx wc{status, &sm.abort_flag, timeout_ns};

    if (tid == 0) {
        sm.abort_flag = 0;
        for (int s = 0; s < AP_STAGES; ++s) {
            mbar_init(smem_addr(&sm.q_full[s]), 1);
            mbar_init(smem_addr(&sm.q_empty[s]), 1);
            mbar_init(smem_addr(&sm.phi_done[s]), PHI_THREADS);
        }
        for (int d = 0; d < D_BUFS; ++d) {
            mbar_init(smem_addr(&sm.mma_done[d]), 1);
            mbar_init(smem_addr(&sm.d_free[d]), EPI_THREADS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_addr(&sm.b_free[i]), 1);
            mbar_init(smem_addr(&sm.bvec_ready[i]), 128);
            mbar_init(smem_addr(&sm.bvec_free[i]), EPI_THREADS);
        }
        mbar_init(smem_addr(&sm.drain), 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
    }
    if (warp == 1) tmem_alloc(smem_addr(&sm.tmem_base), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    auto head_of = [&](int it) { return static_cast<int>((first + it) / Tn); };

    if (warp == 0) {
        if (lane == 0) {
            // =============================================== producer ====
            uint32_t issued = 0, consumed_par = 0, issued_mask = 0;
            bool ok = true;
            for (int it = 0; it < cnt && ok; ++it) {
                const int s = it % AP_STAGES;
                const uint32_t use = static_cast<uint32_t>(it / AP_STAGES);
                if (!mbar_wait_sleep(smem_addr(&sm.q_empty[s]), (use & 1) ^ 1, wc, 20000)) { ok = false; break; }
                const long long item = first + it;
                const int h = static_cast<int>(item / Tn), t = static_cast<int>(item % Tn);
                mbar_arrive_expect_tx(smem_addr(&sm.q_full[s]), TILE_BYTES);
                tma_load_3d(smem_addr(sm.q[s]), &tm_q, smem_addr(&sm.q_full[s]), 0, t * TILE, h);
                issued_mask |= 1u << s;
                consumed_par = (consumed_par & ~(1u << s)) | ((use & 1u) << s);
                ++issued;
            }
            // leave no TMA write in flight (bounded, even after an abort)
            volatile int no_abort = 0;
            const WaitCtx w2{status, &no_abort, drain_timeout_ns(timeout_ns)};
            for (int s = 0; s < AP_STAGES; ++s)
                if ((issued_mask >> s) & 1u) mbar_wait(smem_addr(&sm.q_full[s]), (consumed_par >> s) & 1u, w2);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ================================================= MMA issuer ====
            constexpr uint32_t IDESC = idesc_bf16(128, BN_ROWS, 0, 0);
            int h_prev = -1, nb = -1;  // head of the previous item, builds seen so far - 1
            bool ok = true;
            for (int it = 0; it < cnt && ok; ++it) {
                const int h = head_of(it);
                if (h != h_prev) {
                    if (nb >= 0) umma_commit(smem_addr(&sm.b_free[nb & 1]));  // the previous head's B is done with
                    ++nb;
                    h_prev = h;
                }
                const int s = it % AP_STAGES, d = it % D_BUFS;
                const uint32_t use = static_cast<uint32_t>(it / AP_STAGES), du = static_cast<uint32_t>(it / D_BUFS);
                if (!mbar_wait_sleep(smem_addr(&sm.phi_done[s]), use & 1, wc, 20000)) { ok = false; break; }
                if (!mbar_wait_sleep(smem_addr(&sm.d_free[d]), (du & 1) ^ 1, wc, 20000)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = smem_addr(sm.q[s]);
                const uint32_t b0 = smem_addr(sm.bop[nb & 1]);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(a0 + kk * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(b0 + kk * 32, 16, 1024);
                    umma_ss(tmem + d * 128, ad, bd, IDESC, kk > 0 ? 1u : 0u);
                }
                umma_commit(smem_addr(&sm.mma_done[d]));
                umma_commit(smem_addr(&sm.q_empty[s]));
            }
            // no MMA may still run when TMEM is released
            volatile int no_abort = 0;
            const WaitCtx w2{status, &no_abort, drain_timeout_ns(timeout_ns)};
            umma_commit(smem_addr(&sm.drain));
            mbar_wait(smem_addr(&sm.drain), 0, w2);
        }
        __syncwarp();
    } else if (warp >= 2 && warp < 6) {
        // ======================================= phi and per-head operands ====
        // Every thread runs every iteration (after an abort it skips the waits
        // and the work but keeps the builders' named barriers matched).
        const int t = tid - 64;           // builder and phi index (warps 2..5)
        int h_prev = -1, nb = -1;
        bool ok = true;
        for (int it = 0; it < cnt; ++it) {
            const int h = head_of(it);
            if (h != h_prev) {
                ++nb;
                h_prev = h;
                const int hb = nb & 1;
                // bop / bvec [hb] were last used by the head two builds ago: its MMAs
                // and its epilogue must be done with them
                if (ok && nb >= 2 && !mbar_wait(smem_addr(&sm.b_free[hb]), ((nb - 2) >> 1) & 1, wc)) ok = false;
                if (ok && nb >= 2 && !mbar_wait(smem_addr(&sm.bvec_free[hb]), ((nb - 2) >> 1) & 1, wc)) ok = false;
                // B operand of head h, K-major, 128-byte swizzle: rows n < 64 hold
                // ((S - z c^T) A)[:, n], row 64 holds z, rows 65..79 zero; the bias
                // becomes b' = c A + b.  Centring on c = 1^T S / 1^T z (the output
                // for phi(q) = 1) is an exact identity (phi(q) z c^T / (phi(q) . z)
                // = c^T) that keeps the bf16 operand small, so rounding it does not
                // cancel against b'.
                uint8_t* bo = sm.bop[hb];
                const float* Sh = S + static_cast<size_t>(h) * HD * HD;
                const float* zh = z + static_cast<size_t>(h) * HD;
                const float* Ah = A ? A + static_cast<size_t>(h) * HD * HD : nullptr;
                if (ok && t < HD) {
                    float cs = 0.f, zs = 0.f;
                    for (int k = 0; k < HD; ++k) {
                        cs += __ldg(Sh + k * HD + t);
                        zs += __ldg(zh + k);
                    }
                    sm.cvec[t] = cs / zs;
                }
                named_bar_sync(PHI_BAR, 128);
                if (ok && t < HD) {
                    float ca = 0.f;
                    for (int m = 0; m < HD; ++m) ca = fmaf(sm.cvec[m], Ah ? __ldg(Ah + m * HD + t) : (m == t ? 1.f : 0.f), ca);
                    sm.bvec[hb][t] = ca + (bias ? bias[static_cast<size_t>(h) * HD + t] : 0.f);
                }
                if (ok) {
                    const int ncol = t & 63;       // output column n
                    const int kpart = t >> 6;      // rows k in [32 kpart, 32 kpart + 32)
                    float acol[HD];
#pragma unroll
                    for (int m = 0; m < HD; ++m) acol[m] = Ah ? __ldg(Ah + m * HD + ncol) : (m == ncol ? 1.f : 0.f);
                    for (int kq = 0; kq < 32; kq += 2) {
                        float v2[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int k = kpart * 32 + kq + u;
                            const float* srow = Sh + k * HD;
                            const float zk = __ldg(zh + k);
                            float acc = 0.f;
#pragma unroll
                            for (int m = 0; m < HD; ++m) acc = fmaf(fmaf(-zk, sm.cvec[m], __ldg(srow + m)), acol[m], acc);
                            v2[u] = acc;
                        }
                        const int k = kpart * 32 + kq;  // even: both land in one 32-bit word
                        const int off = ncol * 128 + ((((k >> 3) ^ (ncol & 7))) << 4) + (k & 7) * 2;
                        *reinterpret_cast<uint32_t*>(bo + off) = pack_bf16x2(v2[0], v2[1]);
                    }
                    for (int e = t; e < 16 * HD / 2; e += 128) {
                        // rows 64..79: z then zeros, two values per word
                        const int rr = 64 + e / (HD / 2);
                        const int k = (e % (HD / 2)) * 2;
                        const float a = rr == 64 ? __ldg(zh + k) : 0.f;
                        const float b2 = rr == 64 ? __ldg(zh + k + 1) : 0.f;
                        const int off = rr * 128 + ((((k >> 3) ^ (rr & 7))) << 4) + (k & 7) * 2;
                        *reinterpret_cast<uint32_t*>(bo + off) = pack_bf16x2(a, b2);
                    }
                }
                mbar_arrive(smem_addr(&sm.bvec_ready[hb]));  // bvec [hb] (written by t < 64) is in
                named_bar_sync(PHI_BAR, 128);  // cvec is reused by the next build
            }
            // phi in place on this tile (the whole 16 KB, 128 bytes per thread pass)
            const int s = it % AP_STAGES;
            const uint32_t use = static_cast<uint32_t>(it / AP_STAGES);
            if (ok && !mbar_wait(smem_addr(&sm.q_full[s]), use & 1, wc)) ok = false;
            if (ok) {
                // 1,024 16-byte chunks over 192 threads: all loads, then phi, then stores
                uint8_t* qt = sm.q[s];
                constexpr int PER = (TILE * 8 + PHI_THREADS - 1) / PHI_THREADS;
                uint4 v[PER];
#pragma unroll
                for (int u = 0; u < PER; ++u) {
                    const int c = t + u * PHI_THREADS;
                    if (c < TILE * 8) v[u] = *reinterpret_cast<const uint4*>(qt + c * 16);
                }
#pragma unroll
                for (int u = 0; u < PER; ++u) {
                    const int c = t + u * PHI_THREADS;
                    if (c < TILE * 8) {
                        *reinterpret_cast<uint4*>(qt + c * 16) = make_uint4(phi_bf16x2(v[u].x), phi_bf16x2(v[u].y),
                                                                            phi_bf16x2(v[u].z), phi_bf16x2(v[u].w));
                    }
                }
            }
            fence_proxy_async_smem();  // the MMA reads phi(Q) and B through the async proxy
            mbar_arrive(smem_addr(&sm.phi_done[s]));
        }
    } else if (warp >= 6) {
        // ================================================== epilogue ====
        // Each thread writes its row into a 128-byte-swizzled staging tile (no
        // bank conflicts); one thread then stores the tile with TMA (rows past
        // n_q are not written).  Every thread runs every iteration (after an
        // abort it skips the waits and the work but keeps the named barriers
        // matched).
        const int row = (warp & 3) * 32 + lane;
        const int hf = (warp - 6) >> 2;  // column half of the row
        const int et = tid - 192;
        const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
        int h_prev = -1, nb = -1;
        bool ok = true;
        uint64_t bv2[16];  // this thread's 32 bias values (columns 32 hf ..), as fp32 pairs
        for (int it = 0; it < cnt; ++it) {
            const long long item = first + it;
            const int h = static_cast<int>(item / Tn), t = static_cast<int>(item % Tn);
            if (h != h_prev) {
                if (nb >= 0) mbar_arrive(smem_addr(&sm.bvec_free[nb & 1]));  // done with the previous head's bvec
                ++nb;
                h_prev = h;
                if (ok && !mbar_wait(smem_addr(&sm.bvec_ready[nb & 1]), (nb >> 1) & 1, wc)) ok = false;
                if (ok) {
                    const uint2* bsrc = reinterpret_cast<const uint2*>(sm.bvec[nb & 1]) + 16 * hf;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const uint2 v = bsrc[q];
                        bv2[q] = f2_pack(__uint_as_float(v.x), __uint_as_float(v.y));
                    }
                }
            }
            const int d = it % D_BUFS, ob = it & 1;
            const uint32_t du = static_cast<uint32_t>(it / D_BUFS);
            // the store from this staging buffer two tiles ago has read it
            if (et == 0) bulk_wait_group_read<1>();
            named_bar_sync(EPI_BAR, EPI_THREADS);
            if (ok && !mbar_wait(smem_addr(&sm.mma_done[d]), du & 1, wc)) ok = false;
            if (ok) {
                tc_fence_after();
                uint32_t r[32], den;
                const uint32_t ta = tmem + lane_addr + d * 128;
                tmem_ld32(ta + 32 * hf, r);
                asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(den) : "r"(ta + 64));
                tmem_wait_ld_dep(r);
                asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(den)::"memory");
                tc_fence_before();
                mbar_arrive(smem_addr(&sm.d_free[d]));
                const float inv = 1.f / __uint_as_float(den);
                uint8_t* orow = sm.ost[ob] + row * 128;
                const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int c = 4 * hf + cc;
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint64_t o2 = f2_fma(f2_pack(__uint_as_float(r[cc * 8 + 2 * e]), __uint_as_float(r[cc * 8 + 2 * e + 1])),
                                                   inv2, bv2[cc * 4 + e]);
                        float o0, o1;
                        f2_unpack(o2, o0, o1);
                        pk[e] = pack_bf16x2(o0, o1);
                    }
                    *reinterpret_cast<uint4*>(orow + ((c ^ (row & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            fence_proxy_async_smem();  // the TMA store reads the tile through the async proxy
            named_bar_sync(EPI_BAR, EPI_THREADS);
            if (et == 0 && ok) {
                tma_store_3d(&tm_o, smem_addr(sm.ost[ob]), 0, t * TILE, h);
                bulk_commit_group();
            }
        }
        if (et == 0) bulk_wait_group<0>();  // every store done before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// fp32 output on the CUDA cores, for calibration-sized row sets: one thread
// per query row, (S - z c^T), z and A staged in shared memory in fp32,
//   x_c = phi(q) (S - z c^T) / (phi(q) . z)   (= linear output - c)
//   o   = x_c A + (c A + b)
// with c = 1^T S / 1^T z, the same centring as the tensor-core path.
__global__ void __launch_bounds__(128)
linear_apply_f32_kernel(const uint16_t* __restrict__ Q, int heads, long long n_q, const float* __restrict__ S,
                        const float* __restrict__ z, const float* __restrict__ A,
                        const float* __restrict__ bias, float* __restrict__ O) {
    __shared__ float sc[HD][HD];      // S - z c^T
    __shared__ float am[HD][HD + 1];  // A (identity when absent)
    __shared__ float zz[HD], cc[HD], bb[HD];
    const int h = blockIdx.y;
    const int tid = threadIdx.x;
    const float* Sh = S + static_cast<size_t>(h) * HD * HD;
    const float* zh = z + static_cast<size_t>(h) * HD;
    const float* Ah = A ? A + static_cast<size_t>(h) * HD * HD : nullptr;
    if (tid < HD) {
        float cs = 0.f, zs = 0.f;
        for (int k = 0; k < HD; ++k) {
            cs += Sh[k * HD + tid];
            zs += zh[k];
        }
        cc[tid] = cs / zs;
        zz[tid] = zh[tid];
    }
    for (int e = tid; e < HD * HD; e += blockDim.x) {
        const int m = e / HD, n = e % HD;
        am[m][n] = Ah ? Ah[e] : (m == n ? 1.f : 0.f);
    }
    __syncthreads();
    for (int e = tid; e < HD * HD; e += blockDim.x) {
        const int k = e / HD, n = e % HD;
        sc[k][n] = fmaf(-zz[k], cc[n], Sh[e]);
    }
    if (tid < HD) {
        float ca = 0.f;
        for (int m = 0; m < HD; ++m) ca = fmaf(cc[m], am[m][tid], ca);
        bb[tid] = ca + (bias ? bias[static_cast<size_t>(h) * HD + tid] : 0.f);
    }
    __syncthreads();
    const long long row = static_cast<long long>(blockIdx.x) * blockDim.x + tid;
    if (row >= n_q) return;
    const uint16_t* qr = Q + (static_cast<long long>(h) * n_q + row) * HD;
    float f[HD];
    float den = 0.f;
#pragma unroll
    for (int c8 = 0; c8 < HD / 8; ++c8) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(qr) + c8);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            f[c8 * 8 + 2 * e] = phi(bf16_lo(w[e]));
            f[c8 * 8 + 2 * e + 1] = phi(bf16_hi(w[e]));
        }
    }
#pragma unroll
    for (int k = 0; k < HD; ++k) den = fmaf(f[k], zz[k], den);
    const float inv = 1.f / den;
    float xc[HD];
#pragma unroll 4
    for (int n = 0; n < HD; ++n) {
        float u = 0.f;
#pragma unroll
        for (int k = 0; k < HD; ++k) u = fmaf(f[k], sc[k][n], u);
        xc[n] = u * inv;
    }
    float* orow = O + (static_cast<long long>(h) * n_q + row) * HD;
#pragma unroll 4
    for (int n = 0; n < HD; ++n) {
        float o = bb[n];
#pragma unroll
        for (int m = 0; m < HD; ++m) o = fmaf(xc[m], am[m][n], o);
        orow[n] = o;
    }
}

}  // namespace lin
}  // namespace zb

using namespace zb;

extern "C" size_t zb_linear_state_workspace_bytes(int32_t heads, int64_t n_tokens, int32_t head_dim) {
    if (heads < 1 || n_tokens < 1 || head_dim != 64) return 0;
    return lin::state_ws_bytes(heads, n_tokens);
}

extern "C" zb_status zb_linear_state(const uint16_t* K, const uint16_t* V, int32_t heads,
                                     int64_t n_tokens, int32_t head_dim, float* S, float* z,
                                     void* ws, size_t ws_bytes, void* stream) {
    if (heads < 1 || n_tokens < 1) return ZB_ERR_SHAPE;
    if (head_dim != 64) return ZB_ERR_UNSUPPORTED;
    if (n_tokens > (1ll << 31) - 256) return ZB_ERR_UNSUPPORTED;
    if (!K || !V || !S || !z) return ZB_ERR_NULL;
    if (!aligned16(K) || !aligned16(V) || !aligned16(S) || !aligned16(z) || !aligned16(ws)) return ZB_ERR_ALIGN;
    const size_t need = lin::state_ws_bytes(heads, n_tokens);
    if (!ws || ws_bytes < need) return ZB_ERR_WORKSPACE;
    DeviceInfo dev;
    zb_status e = current_device(&dev);
    if (e != ZB_OK) return e;
    CUtensorMap mk, mv;
    if ((e = make_map_bf16_3d(&mk, K, 64, n_tokens, heads, lin::TILE)) != ZB_OK) return e;
    if ((e = make_map_bf16_3d(&mv, V, 64, n_tokens, heads, lin::TILE)) != ZB_OK) return e;
    const lin::StateGeom geo = lin::state_geom(heads, n_tokens);
    const size_t smem = sizeof(lin::StateSmem) + 1024;
    if (cudaFuncSetAttribute(lin::linear_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return ZB_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* part = static_cast<float*>(ws);
    lin::linear_state_kernel<<<geo.pairs * geo.chunks, lin::ST_THREADS, smem, st>>>(
        mk, mv, heads, n_tokens, geo, part, dev.status, wait_timeout_ns());
    if (cudaGetLastError() != cudaSuccess) return ZB_ERR_CUDA;
    lin::linear_state_reduce_kernel<<<heads, 256, 0, st>>>(part, heads, geo, S, z);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}

extern "C" size_t zb_key_mean_workspace_bytes(int32_t heads, int64_t n_tokens, int32_t head_dim) {
    if (heads < 1 || n_tokens < 1 || head_dim != 64) return 0;
    return static_cast<size_t>(heads) * lin::key_mean_chunks(heads, n_tokens) * lin::HD * sizeof(double);
}

extern "C" zb_status zb_key_mean(const uint16_t* K, int32_t heads, int64_t n_tokens, int32_t head_dim,
                                 float* mu, void* ws, size_t ws_bytes, void* stream) {
    if (heads < 1 || n_tokens < 1) return ZB_ERR_SHAPE;
    if (head_dim != 64) return ZB_ERR_UNSUPPORTED;
    if (heads > 65535 || n_tokens > (1ll << 31) - 256) return ZB_ERR_UNSUPPORTED;
    if (!K || !mu) return ZB_ERR_NULL;
    if (!aligned16(K) || !aligned16(mu) || !aligned16(ws)) return ZB_ERR_ALIGN;
    const size_t need = zb_key_mean_workspace_bytes(heads, n_tokens, head_dim);
    if (!ws || ws_bytes < need) return ZB_ERR_WORKSPACE;
    DeviceInfo dev;
    zb_status e = current_device(&dev);
    if (e != ZB_OK) return e;
    const int chunks = lin::key_mean_chunks(heads, n_tokens);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    double* part = static_cast<double*>(ws);
    lin::key_sum_kernel<<<dim3(static_cast<unsigned>(chunks), static_cast<unsigned>(heads)), lin::KM_THREADS, 0, st>>>(
        K, n_tokens, chunks, part);
    if (cudaGetLastError() != cudaSuccess) return ZB_ERR_CUDA;
    lin::key_mean_reduce_kernel<<<heads, lin::HD, 0, st>>>(part, chunks, n_tokens, mu);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}

extern "C" zb_status zb_linear_state_centered(const uint16_t* K, const uint16_t* V, const float* key_mean,
                                              int32_t heads, int64_t n_tokens, int32_t head_dim, float* S,
                                              float* z, void* ws, size_t ws_bytes, void* stream) {
    if (heads < 1 || n_tokens < 1) return ZB_ERR_SHAPE;
    if (head_dim != 64) return ZB_ERR_UNSUPPORTED;
    if (n_tokens > (1ll << 31) - 256) return ZB_ERR_UNSUPPORTED;
    if (!K || !V || !key_mean || !S || !z) return ZB_ERR_NULL;
    if (!aligned16(K) || !aligned16(V) || !aligned16(key_mean) || !aligned16(S) || !aligned16(z) ||
        !aligned16(ws))
        return ZB_ERR_ALIGN;
    const size_t need = lin::state_ws_bytes(heads, n_tokens);
    if (!ws || ws_bytes < need) return ZB_ERR_WORKSPACE;
    DeviceInfo dev;
    zb_status e = current_device(&dev);
    if (e != ZB_OK) return e;
    CUtensorMap mk, mv;
    if ((e = make_map_bf16_3d(&mk, K, 64, n_tokens, heads, lin::TILE)) != ZB_OK) return e;
    if ((e = make_map_bf16_3d(&mv, V, 64, n_tokens, heads, lin::TILE)) != ZB_OK) return e;
    const lin::StateGeom geo = lin::state_geom(heads, n_tokens);
    const size_t smem = sizeof(lin::StateSmem) + 1024;
    if (cudaFuncSetAttribute(lin::linear_state_centered_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return ZB_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* part = static_cast<float*>(ws);
    lin::linear_state_centered_kernel<<<geo.pairs * geo.chunks, lin::ST_THREADS, smem, st>>>(
        mk, mv, heads, n_tokens, geo, part, dev.status, wait_timeout_ns(), key_mean);
    if (cudaGetLastError() != cudaSuccess) return ZB_ERR_CUDA;
    lin::linear_state_reduce_kernel<<<heads, 256, 0, st>>>(part, heads, geo, S, z);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}

extern "C" zb_status zb_linear_apply(const uint16_t* Q, int32_t heads, int64_t n_q,
                                     int32_t head_dim, const float* S, const float* z,
                                     const float* A, const float* b, void* O, int32_t out_fp32,
                                     void* stream) {
    if (heads < 1 || n_q < 1) return ZB_ERR_SHAPE;
    if (head_dim != 64) return ZB_ERR_UNSUPPORTED;
    if (n_q > (1ll << 31) - 256) return ZB_ERR_UNSUPPORTED;
    if (!Q || !S || !z || !O) return ZB_ERR_NULL;
    if (!aligned16(Q) || !aligned16(S) || !aligned16(z) || !aligned16(A) || !aligned16(b) || !aligned16(O))
        return ZB_ERR_ALIGN;
    DeviceInfo dev;
    zb_status e = current_device(&dev);
    if (e != ZB_OK) return e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (out_fp32) {
        const long long blocks = (n_q + 127) / 128;
        if (blocks > 0x7FFFFFFFll || heads > 65535) return ZB_ERR_UNSUPPORTED;
        lin::linear_apply_f32_kernel<<<dim3(static_cast<unsigned>(blocks), heads), 128, 0, st>>>(
            Q, heads, n_q, S, z, A, b, static_cast<float*>(O));
        return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
    }
    CUtensorMap mq, mo;
    if ((e = make_map_bf16_3d(&mq, Q, 64, n_q, heads, lin::TILE)) != ZB_OK) return e;
    if ((e = make_map_bf16_3d(&mo, O, 64, n_q, heads, lin::TILE)) != ZB_OK) return e;
    const size_t smem = sizeof(lin::ApplySmem) + 1024;
    if (cudaFuncSetAttribute(lin::linear_apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return ZB_ERR_CUDA;
    const long long items = static_cast<long long>(heads) * ((n_q + lin::TILE - 1) / lin::TILE);
    const long long grid = items < dev.sm_count ? items : dev.sm_count;
    lin::linear_apply_kernel<<<static_cast<unsigned>(grid), lin::AP_THREADS, smem, st>>>(
        mq, mo, heads, n_q, S, z, A, b, dev.status, wait_timeout_ns());
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}

// ==================================================== the whole stage ====
// zb_linear_attn = zb_linear_state + zb_linear_apply in one call; the state S,
// z and the state partials live in the caller's workspace:
//   [S: H d d fp32][z: H d fp32][partials], each part 256-byte aligned.
namespace zb {
namespace lin {
static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
static size_t attn_s_bytes(int heads) { return align256(size_t(heads) * 64 * 64 * sizeof(float)); }
static size_t attn_z_bytes(int heads) { return align256(size_t(heads) * 64 * sizeof(float)); }
}  // namespace lin
}  // namespace zb

extern "C" size_t zb_linear_attn_workspace_bytes(int32_t heads, int64_t n_tokens, int32_t head_dim) {
    if (heads < 1 || n_tokens < 1 || head_dim != 64) return 0;
    return lin::attn_s_bytes(heads) + lin::attn_z_bytes(heads) + lin::align256(lin::state_ws_bytes(heads, n_tokens));
}

extern "C" zb_status zb_linear_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int32_t heads,
                                    int64_t n_tokens, int32_t head_dim, const float* A, const float* b,
                                    uint16_t* O, void* ws, size_t ws_bytes, void* stream) {
    if (heads < 1 || n_tokens < 1) return ZB_ERR_SHAPE;
    if (head_dim != 64) return ZB_ERR_UNSUPPORTED;
    if (!Q || !O) return ZB_ERR_NULL;
    if (!aligned16(Q) || !aligned16(O) || !aligned16(A) || !aligned16(b) || !aligned16(ws)) return ZB_ERR_ALIGN;
    const size_t need = zb_linear_attn_workspace_bytes(heads, n_tokens, head_dim);
    if (!ws || ws_bytes < need) return ZB_ERR_WORKSPACE;
    unsigned char* w = static_cast<unsigned char*>(ws);
    float* S = reinterpret_cast<float*>(w);
    float* z = reinterpret_cast<float*>(w + lin::attn_s_bytes(heads));
    void* part = w + lin::attn_s_bytes(heads) + lin::attn_z_bytes(heads);
    zb_status e = zb_linear_state(K, V, heads, n_tokens, head_dim, S, z, part,
                                  ws_bytes - lin::attn_s_bytes(heads) - lin::attn_z_bytes(heads), stream);
    if (e != ZB_OK) return e;
    return zb_linear_apply(Q, heads, n_tokens, head_dim, S, z, A, b, O, 0, stream);
}

// ======================================= linear state without a workspace ====
// zb_linear_state needs a caller-allocated workspace for the per-CTA partial
// states.  Some callers cannot allocate device memory when they call the
// layer: a serving process whose device memory is reserved up front by
// another framework's allocator, or a latency-critical loop where cudaMalloc
// (which may synchronise the device) is not allowed.  zb_linear_state_static
// gives them the same result without any workspace: the partials live in the
// file-scope array below, a fixed 8 MiB that every GPU which loads this
// library holds until the process exits.
namespace zb {
namespace lin {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_state_scratch[kStaticScratchBytes];

namespace {
std::mutex g_static_mu;
float* g_static_ptr[64] = {};  // device address of g_state_scratch, per device
}  // namespace

// Device address of the scratch array on the current device; looked up once per
// device with that device current (the first call on a device does this).
static zb_status static_scratch(int device, float** out) {
    if (device < 0 || device >= 64) return ZB_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[device]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_state_scratch) != cudaSuccess || p == nullptr) return ZB_ERR_CUDA;
        g_static_ptr[device] = static_cast<float*>(p);
    }
    *out = g_static_ptr[device];
    return ZB_OK;
}

}  // namespace lin
}  // namespace zb

extern "C" size_t zb_linear_state_static_scratch_bytes(void) { return zb::lin::kStaticScratchBytes; }

extern "C" zb_status zb_linear_state_static(const uint16_t* K, const uint16_t* V, int32_t heads,
                                            int64_t n_tokens, int32_t head_dim, float* S, float* z,
                                            void* stream) {
    using namespace zb;
    if (heads < 1 || n_tokens < 1) return ZB_ERR_SHAPE;
    if (head_dim != 64) return ZB_ERR_UNSUPPORTED;
    if (n_tokens > (1ll << 31) - 256) return ZB_ERR_UNSUPPORTED;
    if (!K || !V || !S || !z) return ZB_ERR_NULL;
    if (!aligned16(K) || !aligned16(V) || !aligned16(S) || !aligned16(z)) return ZB_ERR_ALIGN;
    // the partial states of this shape must fit the fixed scratch
    if (lin::state_ws_bytes(heads, n_tokens) > lin::kStaticScratchBytes) return ZB_ERR_UNSUPPORTED;
    DeviceInfo dev;
    zb_status e = current_device(&dev);
    if (e != ZB_OK) return e;
    float* part = nullptr;
    if ((e = lin::static_scratch(dev.device, &part)) != ZB_OK) return e;
    CUtensorMap mk, mv;
    if ((e = make_map_bf16_3d(&mk, K, 64, n_tokens, heads, lin::TILE)) != ZB_OK) return e;
    if ((e = make_map_bf16_3d(&mv, V, 64, n_tokens, heads, lin::TILE)) != ZB_OK) return e;
    const lin::StateGeom geo = lin::state_geom(heads, n_tokens);
    const size_t smem = sizeof(lin::StateSmem) + 1024;
    if (cudaFuncSetAttribute(lin::linear_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return ZB_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // Every CTA writes its whole partial slot (zeros when it has no tokens), so
    // nothing left in the scratch by an earlier call is read.
    lin::linear_state_kernel<<<geo.pairs * geo.chunks, lin::ST_THREADS, smem, st>>>(
        mk, mv, heads, n_tokens, geo, part, dev.status, wait_timeout_ns());
    if (cudaGetLastError() != cudaSuccess) return ZB_ERR_CUDA;
    lin::linear_state_reduce_kernel<<<heads, 256, 0, st>>>(part, heads, geo, S, z);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}
