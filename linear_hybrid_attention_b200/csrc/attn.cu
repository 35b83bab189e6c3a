// Tile-sparse softmax attention with mean-key/value landmarks, and its dense
// special case, on sm_100a tensor cores.
//
// Method (by page title): "Zebra3D: Efficient Hybrid Foundation Models For
// Scalable 3D Reconstruction", Figure 1 (a) caption -- every query tile keeps
// exact softmax over its selected key tiles; each omitted key tile is replaced
// by one landmark token (mean key, mean value).  "Zebra3D speeds up 3D
// reconstruction by up to 7.1x on 1024 frames without training from scratch",
// section "How Zebra3D works" -- only the selected blocks of tokens are
// computed.  A landmark's logit carries + ln(n_j) so that it weighs as much as
// the n_j keys it stands for.
//
// Kernel design (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: Q tile of the work item, then for each step the
//               K and V tile of a selected key tile or a 128-landmark chunk,
//               into a KV_STAGES-deep ring; also the selected-tile bitmap.
//   warp 1      MMA issuer (one lane): S = Q K^T into a double-buffered TMEM S,
//               then O += P V with P read from TMEM (tcgen05 "TS" form).
//   warps 2..5  softmax warpgroup: one thread per query row; loads its S row
//               from TMEM, masks, online softmax in the log2 domain with lazy
//               rescaling of O, writes P (bf16) to TMEM; epilogue O / l.
// A work item is one (head, query tile); items are dealt round-robin so that
// CTAs running at the same time work on neighbouring query tiles of the same
// head and sweep that head's K/V in ascending order together (L2 reuse).
#include <cuda.h>
#include <cuda_runtime.h>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace attn {

constexpr int BM = 128;          // query rows per work item (MMA M)
constexpr int BN = 128;          // keys per step (QK MMA N, PV MMA K)
constexpr int HD = 64;           // head dim
constexpr int KV_STAGES = 4;
constexpr int NUM_THREADS = 192;
constexpr int MAX_TILES = 32768;  // bitmap capacity (key tiles)
constexpr uint32_t TILE_BYTES = BN * HD * 2;  // 16 KB, one 128 x 64 bf16 tile
constexpr uint32_t TMEM_COLS = 512;
// TMEM column map
constexpr uint32_t TM_S0 = 0;     // S buffer 0: 128 fp32 columns
constexpr uint32_t TM_S1 = 128;   // S buffer 1
constexpr uint32_t TM_O = 256;    // O accumulator: 64 fp32 columns
constexpr uint32_t TM_P0 = 320;   // P buffer 0: 128 bf16 packed in 64 columns
constexpr uint32_t TM_P1 = 384;   // P buffer 1

constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: p <= 2^8 before a rescale

struct Smem {
    uint8_t q[2][TILE_BYTES];
    uint8_t k[KV_STAGES][TILE_BYTES];
    uint8_t v[KV_STAGES][TILE_BYTES];
    uint32_t bitmap[2][MAX_TILES / 32];
    uint64_t q_full[2], q_empty[2];
    uint64_t kv_full[KV_STAGES], kv_empty[KV_STAGES];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full[2], p_free[2];
    uint64_t o_free;
    uint64_t bm_full[2], bm_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

struct Params {
    int heads;
    long long n_q, n_kv;
    int tq, tk;        // query / key tile rows (64 or 128)
    int Tq, Tk;        // query / key tile counts
    int n_last;        // keys in the last key tile
    int k;             // selected key tiles per query tile (dense: Tk)
    int dense;         // 1: keep every key tile, no index list
    int use_lm;        // landmarks for unselected tiles
    int lm_chunks;     // ceil(Tk / 128) when landmarks are used, else 0
    float scale_log2;  // softmax scale * log2(e)
    float log2_tk, log2_last;
    long long n_items;
    const int32_t* idx;
    void* O;
    int out_fp32;      // 1: O is fp32, else bf16
    float* lse;
    int* status;
    unsigned long long timeout_ns;
};

__device__ __forceinline__ int steps_of(const Params& p) {
    return p.k + p.lm_chunks;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kb,
                   const __grid_constant__ CUtensorMap tm_vb, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = warp_id();
    const int lane = lane_id();
    const WaitCtx wc{p.status, &sm.abort_flag, p.timeout_ns};
    const int n_steps = steps_of(p);

    // ---------------------------------------------------------- set-up ----
    // Zero the operand buffers once: a 64-row TMA box leaves rows 64..127 of
    // a buffer untouched, and those rows must hold finite values.
    {
        uint4* z = reinterpret_cast<uint4*>(&sm.q[0][0]);
        const int n16 = (2 + 2 * KV_STAGES) * TILE_BYTES / 16;
        for (int i = threadIdx.x; i < n16; i += NUM_THREADS) z[i] = make_uint4(0, 0, 0, 0);
    }
    if (threadIdx.x == 0) {
        sm.abort_flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_addr(&sm.q_full[i]), 1);
            mbar_init(smem_addr(&sm.q_empty[i]), 1);
            mbar_init(smem_addr(&sm.s_full[i]), 1);
            mbar_init(smem_addr(&sm.s_free[i]), 128);
            mbar_init(smem_addr(&sm.p_full[i]), 128);
            mbar_init(smem_addr(&sm.p_free[i]), 1);
            mbar_init(smem_addr(&sm.bm_full[i]), 1);
            mbar_init(smem_addr(&sm.bm_empty[i]), 128);
        }
        for (int i = 0; i < KV_STAGES; ++i) {
            mbar_init(smem_addr(&sm.kv_full[i]), 1);
            mbar_init(smem_addr(&sm.kv_empty[i]), 1);
        }
        mbar_init(smem_addr(&sm.o_free), 128);
        mbar_init(smem_addr(&sm.drain), 1);
        fence_mbar_init();
    }
    fence_proxy_async_smem();
    if (warp == 1) tmem_alloc(smem_addr(&sm.tmem_base), TMEM_COLS);
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        if (p.lm_chunks) {
            tma_prefetch_desc(&tm_kb);
            tma_prefetch_desc(&tm_vb);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ============================================== TMA producer ====
        // Lane 0 does every wait and issues every copy; the warp helps read
        // the index list and build the bitmap.  Each wait's outcome is
        // broadcast so that all lanes leave the loops together.
        const uint32_t FULL = 0xffffffffu;
        long long g = 0;
        int it = 0;
        // per-buffer bit: a load was issued / parity of the last one issued
        uint32_t kv_issued = 0, kv_parity = 0, q_issued = 0, q_parity = 0;
        bool ok = true;
        for (long long item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++it) {
            const int h = static_cast<int>(item / p.Tq);
            const int i = static_cast<int>(item % p.Tq);
            const int32_t* list = p.dense ? nullptr : p.idx + item * static_cast<long long>(p.k);
            // selected-tile bitmap for the landmark steps of this item
            if (p.lm_chunks) {
                const int b = it & 1;
                int w_ok = 1;
                if (lane == 0) w_ok = mbar_wait(smem_addr(&sm.bm_empty[b]), ((it >> 1) & 1) ^ 1, wc);
                if (!__shfl_sync(FULL, w_ok, 0)) { ok = false; break; }
                uint32_t* bm = sm.bitmap[b];
                const int words = (p.Tk + 31) >> 5;
                for (int w = lane; w < words; w += 32) bm[w] = 0u;
                __syncwarp();
                int bad = 0;
                for (int q0 = 0; q0 < p.k; q0 += 32) {
                    const int qq = q0 + lane;
                    const int j = qq < p.k ? list[qq] : 0;
                    int jprev = __shfl_up_sync(FULL, j, 1);
                    if (lane == 0) jprev = (q0 == 0) ? -1 : list[q0 - 1];
                    if (qq < p.k) {
                        if (j < 0 || j >= p.Tk || j <= jprev) bad = 1;
                        else atomicOr(&bm[j >> 5], 1u << (j & 31));
                    }
                }
                if (__any_sync(FULL, bad) && lane == 0) flag_status(p.status, ZB_ERR_INDEX);
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&sm.bm_full[b]));
            }
            // Q tile
            const int qs = it & 1;
            {
                int w_ok = 1;
                if (lane == 0) {
                    w_ok = mbar_wait(smem_addr(&sm.q_empty[qs]), ((it >> 1) & 1) ^ 1, wc);
                    if (w_ok) {
                        const uint32_t bar = smem_addr(&sm.q_full[qs]);
                        mbar_arrive_expect_tx(bar, p.tq * HD * 2);
                        tma_load_3d(smem_addr(sm.q[qs]), &tm_q, bar, 0, i * p.tq, h);
                        q_issued |= 1u << qs;
                        q_parity = (q_parity & ~(1u << qs)) | (((it >> 1) & 1u) << qs);
                    }
                }
                if (!__shfl_sync(FULL, w_ok, 0)) { ok = false; break; }
            }
            // K/V steps
            int jcache = 0;
            for (int st = 0; st < n_steps; ++st) {
                const long long gg = g + st;
                const int s = static_cast<int>(gg % KV_STAGES);
                const uint32_t use = static_cast<uint32_t>(gg / KV_STAGES);
                if (!p.dense && st < p.k && (st & 31) == 0) {
                    const int qq = st + lane;
                    jcache = qq < p.k ? list[qq] : 0;
                }
                int j = st;
                if (!p.dense && st < p.k) j = __shfl_sync(FULL, jcache, st & 31);
                int w_ok = 1;
                if (lane == 0) {
                    w_ok = mbar_wait(smem_addr(&sm.kv_empty[s]), (use & 1) ^ 1, wc);
                    if (w_ok) {
                        const uint32_t bar = smem_addr(&sm.kv_full[s]);
                        if (st < p.k) {
                            j = j < 0 ? 0 : (j >= p.Tk ? p.Tk - 1 : j);
                            mbar_arrive_expect_tx(bar, 2u * p.tk * HD * 2);
                            tma_load_3d(smem_addr(sm.k[s]), &tm_k, bar, 0, j * p.tk, h);
                            tma_load_3d(smem_addr(sm.v[s]), &tm_v, bar, 0, j * p.tk, h);
                        } else {
                            const int c = st - p.k;
                            mbar_arrive_expect_tx(bar, 2u * TILE_BYTES);
                            tma_load_3d(smem_addr(sm.k[s]), &tm_kb, bar, 0, c * BN, h);
                            tma_load_3d(smem_addr(sm.v[s]), &tm_vb, bar, 0, c * BN, h);
                        }
                        kv_issued |= 1u << s;
                        kv_parity = (kv_parity & ~(1u << s)) | ((use & 1u) << s);
                    }
                }
                if (!__shfl_sync(FULL, w_ok, 0)) { ok = false; break; }
            }
            g += n_steps;
        }
        // Leave no TMA write in flight: wait (bounded, even after an abort) for
        // the last load issued into every buffer.
        if (lane == 0) {
            volatile int no_abort = 0;
            const WaitCtx w2{p.status, &no_abort, p.timeout_ns};
            for (int s = 0; s < KV_STAGES; ++s)
                if ((kv_issued >> s) & 1u) mbar_wait(smem_addr(&sm.kv_full[s]), (kv_parity >> s) & 1u, w2);
            for (int s = 0; s < 2; ++s)
                if ((q_issued >> s) & 1u) mbar_wait(smem_addr(&sm.q_full[s]), (q_parity >> s) & 1u, w2);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================================================= MMA issuer ====
        constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, 0, 0);  // Q K-major, K K-major
        constexpr uint32_t IDESC_PV = idesc_bf16(BM, HD, 0, 1);  // P (TMEM), V MN-major
        if (lane == 0) {
            long long g = 0;
            int it = 0;
            bool ok = true;
            for (long long item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++it) {
                const int qs = it & 1;
                if (!mbar_wait(smem_addr(&sm.q_full[qs]), (it >> 1) & 1, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t q_base = smem_addr(sm.q[qs]);
                // S[b] = Q K_s^T for step gg
                auto issue_qk = [&](long long gg) -> bool {
                    const int s = static_cast<int>(gg % KV_STAGES);
                    const uint32_t use = static_cast<uint32_t>(gg / KV_STAGES);
                    const int b = static_cast<int>(gg & 1);
                    const uint32_t buse = static_cast<uint32_t>(gg >> 1);
                    if (!mbar_wait(smem_addr(&sm.kv_full[s]), use & 1, wc)) return false;
                    if (!mbar_wait(smem_addr(&sm.s_free[b]), (buse & 1) ^ 1, wc)) return false;
                    tc_fence_after();
                    const uint32_t k_base = smem_addr(sm.k[s]);
                    const uint32_t d_tmem = tmem + (b ? TM_S1 : TM_S0);
#pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk) {
                        const uint64_t ad = sdesc_sw128(q_base + kk * 32, 16, 1024);
                        const uint64_t bd = sdesc_sw128(k_base + kk * 32, 16, 1024);
                        umma_ss(d_tmem, ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(smem_addr(&sm.s_full[b]));
                    return true;
                };
                if (!issue_qk(g)) { ok = false; break; }
                for (int st = 0; st < n_steps; ++st) {
                    const long long gg = g + st;
                    if (st + 1 < n_steps) {
                        if (!issue_qk(gg + 1)) { ok = false; break; }
                    }
                    if (st + 1 == n_steps) umma_commit(smem_addr(&sm.q_empty[qs]));
                    const int b = static_cast<int>(gg & 1);
                    const uint32_t buse = static_cast<uint32_t>(gg >> 1);
                    if (!mbar_wait(smem_addr(&sm.p_full[b]), buse & 1, wc)) { ok = false; break; }
                    if (st == 0) {
                        if (!mbar_wait(smem_addr(&sm.o_free), (it & 1) ^ 1, wc)) { ok = false; break; }
                    }
                    tc_fence_after();
                    const int s = static_cast<int>(gg % KV_STAGES);
                    const uint32_t v_base = smem_addr(sm.v[s]);
                    const uint32_t p_tmem = tmem + (b ? TM_P1 : TM_P0);
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        const uint64_t bd = sdesc_sw128(v_base + kk * 2048, 0, 1024);
                        umma_ts(tmem + TM_O, p_tmem + kk * 8, bd, IDESC_PV, (st > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(smem_addr(&sm.kv_empty[s]));
                    umma_commit(smem_addr(&sm.p_free[b]));
                }
                g += n_steps;
            }
            // No tcgen05.mma may still run when TMEM is released.
            umma_commit(smem_addr(&sm.drain));
            volatile int no_abort = 0;
            const WaitCtx w2{p.status, &no_abort, p.timeout_ns};
            mbar_wait(smem_addr(&sm.drain), 0, w2);
        }
        __syncwarp();
    } else {
        // ============================================ softmax warpgroup ====
        const int quarter = warp & 3;            // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;     // query row within the tile
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        long long g = 0;
        int it = 0;
        bool ok = true;
        for (long long item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++it) {
            const int h = static_cast<int>(item / p.Tq);
            const int i = static_cast<int>(item % p.Tq);
            // valid columns of the last selected tile (only the last key tile is ragged)
            int last_valid = p.tk;
            if (p.k > 0) {
                const int jl = p.dense ? p.Tk - 1 : p.idx[item * static_cast<long long>(p.k) + p.k - 1];
                if (jl == p.Tk - 1) last_valid = p.n_last;
            }
            const uint32_t* bm = sm.bitmap[it & 1];
            if (p.lm_chunks) {
                if (!mbar_wait(smem_addr(&sm.bm_full[it & 1]), (it >> 1) & 1, wc)) { ok = false; break; }
            }
            float m = -INFINITY;  // running max of the log2-domain logits (lazy)
            float l = 0.f;        // running sum of 2^(x - m)
            for (int st = 0; st < n_steps; ++st) {
                const long long gg = g + st;
                const int b = static_cast<int>(gg & 1);
                const uint32_t buse = static_cast<uint32_t>(gg >> 1);
                if (!mbar_wait(smem_addr(&sm.s_full[b]), buse & 1, wc)) { ok = false; break; }
                tc_fence_after();
                float x[BN];
                {
                    uint32_t raw[BN];
                    const uint32_t sa = tmem + lane_addr + (b ? TM_S1 : TM_S0);
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c) tmem_ld32(sa + c * 32, sub32(raw, c * 32));
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c) tmem_wait_ld_dep(sub32(raw, c * 32));
#pragma unroll
                    for (int e = 0; e < BN; ++e) x[e] = __uint_as_float(raw[e]);
                }
                tc_fence_before();
                mbar_arrive(smem_addr(&sm.s_free[b]));
                // ---- row max (tree of 3-input max; no long dependency chain)
                // Selected tiles: max of the raw scores, scaled afterwards
                // (scale > 0).  Landmark chunks: x = s * scale + bias first,
                // bias = log2(n_j), or -inf for selected / out-of-range tiles.
                const bool is_lm = st >= p.k;
                const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
                if (!is_lm) {
                    const int valid = (st == p.k - 1) ? last_valid : p.tk;
                    if (valid < BN) {
#pragma unroll
                        for (int e = 0; e < BN; ++e)
                            if (e >= valid) x[e] = -INFINITY;
                    }
                } else {
                    const int j0 = (st - p.k) * BN;
#pragma unroll
                    for (int w = 0; w < BN / 32; ++w) {
                        const int jw = j0 + w * 32;
                        uint32_t bits = (jw < p.Tk) ? bm[jw >> 5] : 0xFFFFFFFFu;
                        if (jw + 32 > p.Tk) {  // the chunk runs past the last tile
                            const int keep = p.Tk - jw;
                            bits |= keep <= 0 ? 0xFFFFFFFFu : (0xFFFFFFFFu << keep);
                        }
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int j = jw + e;
                            float b0 = (j == p.Tk - 1) ? p.log2_last : p.log2_tk;
                            float b1 = (j + 1 == p.Tk - 1) ? p.log2_last : p.log2_tk;
                            if ((bits >> e) & 1u) b0 = -INFINITY;
                            if ((bits >> (e + 1)) & 1u) b1 = -INFINITY;
                            float v0, v1;
                            f2_unpack(f2_fma(f2_pack(x[w * 32 + e], x[w * 32 + e + 1]), c2, f2_pack(b0, b1)), v0, v1);
                            x[w * 32 + e] = v0;
                            x[w * 32 + e + 1] = v1;
                        }
                    }
                }
                float mx;
                {
                    float g[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float t = fmax3(x[16 * q], x[16 * q + 1], x[16 * q + 2]);
#pragma unroll
                        for (int e = 3; e < 15; e += 2) t = fmax3(t, x[16 * q + e], x[16 * q + e + 1]);
                        g[q] = fmaxf(t, x[16 * q + 15]);
                    }
                    mx = fmax3(fmax3(g[0], g[1], g[2]), fmax3(g[3], g[4], g[5]), fmaxf(g[6], g[7]));
                }
                if (!is_lm) mx *= p.scale_log2;
                // ---- lazy rescale: keep the old max unless the new one exceeds it by > 8
                const float m_new = fmaxf(m, mx);
                const bool rescale = m_new > m + RESCALE_THRESHOLD;
                float alpha = 1.f;
                if (rescale) {
                    alpha = (m == -INFINITY) ? 0.f : ex2(m - m_new);
                    m = m_new;
                    l *= alpha;
                }
                const float msub = (m == -INFINITY) ? 0.f : m;
                // ---- p = 2^(x - m): 3 of every 8 pairs on the FMA pipes, the
                // rest on MUFU; packed fp32x2 arithmetic; 4 independent sums
                uint32_t pk[BN / 2];
                const uint64_t nm2 = f2_pack(-msub, -msub);
                uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int q = 0; q < BN / 2; ++q) {
                    const uint64_t xin = f2_pack(x[2 * q], x[2 * q + 1]);
                    const uint64_t xs = is_lm ? f2_add(xin, nm2) : f2_fma(xin, c2, nm2);
                    uint64_t pv;
                    if ((q & 7) < 3) {
                        pv = f2_exp2_poly(xs);
                    } else {
                        float a0, a1;
                        f2_unpack(xs, a0, a1);
                        pv = f2_pack(ex2(a0), ex2(a1));
                    }
                    acc[q & 3] = f2_add(acc[q & 3], pv);
                    float p0, p1;
                    f2_unpack(pv, p0, p1);
                    pk[q] = pack_bf16x2(p0, p1);
                }
                {
                    float s0, s1, s2, s3;
                    f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), s0, s1);
                    (void)s2;
                    (void)s3;
                    l += s0 + s1;
                }
                // P buffer b is free once PV of step gg-2 is done
                if (!mbar_wait(smem_addr(&sm.p_free[b]), (buse & 1) ^ 1, wc)) { ok = false; break; }
                if (rescale && st > 0) {
                    // O must hold every PV up to step gg-1 before it is rescaled
                    const long long gp = gg - 1;
                    if (!mbar_wait(smem_addr(&sm.p_free[gp & 1]), static_cast<uint32_t>(gp >> 1) & 1, wc)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint32_t ro[HD];
                    const uint32_t oa = tmem + lane_addr + TM_O;
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) tmem_ld32(oa + c * 32, sub32(ro, c * 32));
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) tmem_wait_ld_dep(sub32(ro, c * 32));
#pragma unroll
                    for (int e = 0; e < HD; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * alpha);
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) tmem_st32(oa + c * 32, sub32(ro, c * 32));
                    tmem_wait_st();
                }
                {
                    const uint32_t pa = tmem + lane_addr + (b ? TM_P1 : TM_P0);
#pragma unroll
                    for (int c = 0; c < BN / 64; ++c) tmem_st32(pa + c * 32, sub32(pk, c * 32));
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_addr(&sm.p_full[b]));
            }
            if (!ok) break;
            if (p.lm_chunks) mbar_arrive(smem_addr(&sm.bm_empty[it & 1]));
            // ------------------------------------------------ epilogue ----
            const long long gl = g + n_steps - 1;
            if (!mbar_wait(smem_addr(&sm.p_free[gl & 1]), static_cast<uint32_t>(gl >> 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
            float o[HD];
            {
                uint32_t ro[HD];
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) tmem_ld32(tmem + lane_addr + TM_O + c * 32, sub32(ro, c * 32));
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) tmem_wait_ld_dep(sub32(ro, c * 32));
#pragma unroll
                for (int e = 0; e < HD; ++e) o[e] = __uint_as_float(ro[e]);
            }
            tc_fence_before();
            mbar_arrive(smem_addr(&sm.o_free));
            const long long qrow = static_cast<long long>(i) * p.tq + row;
            if (row < p.tq && qrow < p.n_q) {
                const float inv = 1.f / l;
                const long long orow = (static_cast<long long>(h) * p.n_q + qrow) * HD;
                if (p.out_fp32) {
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.O) + orow);
#pragma unroll
                    for (int c = 0; c < HD / 4; ++c)
                        dst[c] = make_float4(o[c * 4] * inv, o[c * 4 + 1] * inv, o[c * 4 + 2] * inv, o[c * 4 + 3] * inv);
                } else {
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.O) + orow);
#pragma unroll
                    for (int c = 0; c < HD / 8; ++c) {
                        uint4 v;
                        v.x = pack_bf16x2(o[c * 8 + 0] * inv, o[c * 8 + 1] * inv);
                        v.y = pack_bf16x2(o[c * 8 + 2] * inv, o[c * 8 + 3] * inv);
                        v.z = pack_bf16x2(o[c * 8 + 4] * inv, o[c * 8 + 5] * inv);
                        v.w = pack_bf16x2(o[c * 8 + 6] * inv, o[c * 8 + 7] * inv);
                        dst[c] = v;
                    }
                }
                if (p.lse) p.lse[static_cast<long long>(h) * p.n_q + qrow] = (m + __log2f(l)) * 0.6931471805599453f;
            }
            g += n_steps;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace attn

static size_t attn_smem_bytes() { return sizeof(attn::Smem) + 1024; }

// Shared launcher of the sparse and dense entry points.
static zb_status launch_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                             const uint16_t* Kb, const uint16_t* Vb, const int32_t* idx, int heads,
                             long long n_q, long long n_kv, int tq, int tk, int k, int dense,
                             int use_lm, float scale, void* O, int out_fp32, float* lse,
                             cudaStream_t st) {
    using namespace attn;
    DeviceInfo dev;
    zb_status e = current_device(&dev);
    if (e != ZB_OK) return e;
    const int Tq = static_cast<int>((n_q + tq - 1) / tq);
    const int Tk = static_cast<int>((n_kv + tk - 1) / tk);
    CUtensorMap mq, mk, mv, mkb, mvb;
    if ((e = make_map_bf16_3d(&mq, Q, HD, n_q, heads, tq)) != ZB_OK) return e;
    if ((e = make_map_bf16_3d(&mk, K, HD, n_kv, heads, tk)) != ZB_OK) return e;
    if ((e = make_map_bf16_3d(&mv, V, HD, n_kv, heads, tk)) != ZB_OK) return e;
    const int lm_chunks = (use_lm && k < Tk) ? (Tk + BN - 1) / BN : 0;
    if (lm_chunks) {
        if ((e = make_map_bf16_3d(&mkb, Kb, HD, Tk, heads, BN)) != ZB_OK) return e;
        if ((e = make_map_bf16_3d(&mvb, Vb, HD, Tk, heads, BN)) != ZB_OK) return e;
    } else {
        mkb = mk;
        mvb = mv;
    }
    Params p{};
    p.heads = heads;
    p.n_q = n_q;
    p.n_kv = n_kv;
    p.tq = tq;
    p.tk = tk;
    p.Tq = Tq;
    p.Tk = Tk;
    p.n_last = static_cast<int>(n_kv - static_cast<long long>(Tk - 1) * tk);
    p.k = k;
    p.dense = dense;
    p.use_lm = use_lm;
    p.lm_chunks = lm_chunks;
    p.scale_log2 = scale * LOG2E;
    p.log2_tk = log2f(static_cast<float>(tk));
    p.log2_last = log2f(static_cast<float>(p.n_last));
    p.n_items = static_cast<long long>(heads) * Tq;
    p.idx = idx;
    p.O = O;
    p.out_fp32 = out_fp32;
    p.lse = lse;
    p.status = dev.status;
    p.timeout_ns = wait_timeout_ns();
    const size_t smem = attn_smem_bytes();
    cudaError_t ce = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(smem));
    if (ce != cudaSuccess) return ZB_ERR_CUDA;
    const long long grid = p.n_items < dev.sm_count ? p.n_items : dev.sm_count;
    sparse_attn_kernel<<<static_cast<unsigned>(grid), NUM_THREADS, smem, st>>>(mq, mk, mv, mkb, mvb, p);
    return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}

}  // namespace zb

using namespace zb;

extern "C" zb_status zb_tile_sparse_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                         const uint16_t* Kbar_bf16, const uint16_t* Vbar_bf16,
                                         const int32_t* idx, int32_t k, int32_t use_landmarks,
                                         float scale, zb_shape s, uint16_t* O, float* lse,
                                         void* stream) {
    zb_status e = check_shape(s);
    if (e != ZB_OK) return e;
    if (!Q || !K || !V || !O) return ZB_ERR_NULL;
    const long long T = n_tiles(s);
    if (T > attn::MAX_TILES) return ZB_ERR_UNSUPPORTED;
    if (k < 0 || k > T) return ZB_ERR_SHAPE;
    if (k == 0 && !use_landmarks) return ZB_ERR_SHAPE;
    if (k > 0 && !idx) return ZB_ERR_NULL;
    const bool lm = use_landmarks && k < T;
    if (lm && (!Kbar_bf16 || !Vbar_bf16)) return ZB_ERR_NULL;
    if (!(scale > 0.f) || !isfinite(scale)) return ZB_ERR_SHAPE;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(idx) ||
        !aligned16(lse) || (lm && (!aligned16(Kbar_bf16) || !aligned16(Vbar_bf16))))
        return ZB_ERR_ALIGN;
    return launch_attn(Q, K, V, Kbar_bf16, Vbar_bf16, idx, s.heads, s.n_tokens, s.n_tokens, s.tile,
                       s.tile, k, 0, use_landmarks ? 1 : 0, scale, O, 0, lse,
                       static_cast<cudaStream_t>(stream));
}

extern "C" zb_status zb_dense_attn(const uint16_t* Q, int64_t n_q, const uint16_t* K,
                                   const uint16_t* V, int64_t n_kv, int32_t heads,
                                   int32_t head_dim, float scale, void* O, int32_t out_fp32,
                                   float* lse, void* stream) {
    if (heads < 1 || n_q < 1 || n_kv < 1) return ZB_ERR_SHAPE;
    if (head_dim != 64) return ZB_ERR_UNSUPPORTED;
    if (!Q || !K || !V || !O) return ZB_ERR_NULL;
    if (n_q > (1ll << 31) - 256 || n_kv > (1ll << 31) - 256) return ZB_ERR_UNSUPPORTED;
    if (!(scale > 0.f) || !isfinite(scale)) return ZB_ERR_SHAPE;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(lse))
        return ZB_ERR_ALIGN;
    const int Tk = static_cast<int>((n_kv + 127) / 128);
    return launch_attn(Q, K, V, nullptr, nullptr, nullptr, heads, n_q, n_kv, 128, 128, Tk, 1, 0,
                       scale, O, out_fp32 ? 1 : 0, lse, static_cast<cudaStream_t>(stream));
}
