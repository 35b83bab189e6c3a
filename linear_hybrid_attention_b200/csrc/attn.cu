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
// Kernel design: one persistent CTA per SM, 384 threads, two work items in
// flight ("slots").  A work item is one (head, query tile); the CTA's items
// alternate between the slots.  With d = 64 the softmax (16,384 exponentials
// per 128 x 128 tile) costs more than the tile's two MMAs, so both slots'
// softmax warpgroups run at the same time while one warp keeps the tensor core
// fed for both.
//   warp 0      Q and K producer (TMA): Q of each slot's item, then K tiles of
//               the selected key tiles / landmark chunks into a K ring.
//   warp 2      V producer (TMA): the matching V tiles into a separate V ring
//               (K is released after Q K^T, V only after P V).
//   warp 1      MMA issuer (one lane): per slot S = Q K^T into the slot's TMEM
//               S, then O += P V with P read from TMEM (tcgen05 "TS" form).
//   warp 3      checks every index list (range, strictly ascending).
//   warps 4..7  softmax of slot 0, warps 8..11 softmax of slot 1: one thread
//               per query row; log2-domain online softmax with lazy
//               rescaling of O, P (bf16) to TMEM, epilogue O / l.
// A softmax thread reads its S row from TMEM twice in 32-column chunks (once
// for the row max, once for the exponentials): compact code (the instruction
// cache is shared by 12 warps running different roles) and few registers.
// Items are dealt round-robin over CTAs, so CTAs running at the same time work
// on neighbouring query tiles of one head and sweep its K/V in ascending order
// together (L2 reuse).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace attn {

constexpr int BM = 128;          // query rows per work item (MMA M)
constexpr int BN = 128;          // keys per step (QK MMA N, PV MMA K)
constexpr int HD = 64;           // head dim
constexpr int SLOTS = 2;
constexpr int K_STAGES = 6;
constexpr int V_STAGES = 4;
constexpr int NUM_THREADS = 384;
constexpr int MAX_TILES = 32768;
constexpr uint32_t TILE_BYTES = BN * HD * 2;  // 16 KB, one 128 x 64 bf16 tile
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns of slot s start at 256 s: S (128 fp32), P (64 = 128 bf16), O (64 fp32)
constexpr uint32_t SLOT_COLS = 256, TM_S = 0, TM_P = 128, TM_O = 192;

constexpr uint32_t SLEEP_NS = 20000;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: p <= 2^8 before a rescale

struct Smem {
    uint8_t q[SLOTS][TILE_BYTES];
    uint8_t k[K_STAGES][TILE_BYTES];
    uint8_t v[V_STAGES][TILE_BYTES];
    uint64_t q_full[SLOTS], q_empty[SLOTS];
    uint64_t k_full[K_STAGES], k_empty[K_STAGES];
    uint64_t v_full[V_STAGES], v_empty[V_STAGES];
    uint64_t s_full[SLOTS], s_free[SLOTS], p_full[SLOTS], p_free[SLOTS], o_free[SLOTS];
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

// 32 lanes x 16 consecutive 32-bit columns
ZB_DEVINL void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// 2^x of one value on the FMA pipes (see f2_exp2_poly for the method).
ZB_DEVINL float exp2_poly(float x) {
    constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
    constexpr float kC1 = 0.695116758f, kC2 = 0.227644995f, kC3 = 0.0770670399f;
    x = fmaxf(x, -127.f);
    const float t = __fadd_rd(x, kShift);
    const float f = x - (t - kShift);
    float p = fmaf(kC3, f, kC2);
    p = fmaf(p, f, kC1);
    p = fmaf(p, f, 1.f);
    return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

// Shared-memory descriptors of the 128-byte-swizzle operand tiles, split in
// 32-bit halves: the low word holds the start address (>> 4) and LBO, the high
// word SBO = 1024, the tcgen05 version bit and the swizzle mode, which are the
// same for every tile here.  Stepping along a tile only adds to the low word
// (the address field never overflows into LBO: shared memory is < 256 KB).
constexpr uint32_t DESC_HI = (1024u >> 4) | (1u << 14) | (2u << 29);
ZB_DEVINL uint32_t desc_lo(uint32_t saddr, uint32_t lbo) { return ((saddr >> 4) & 0x3FFFu) | ((lbo >> 4) << 16); }

// D[tmem] (+)= A[smem] * B[smem], descriptors given by their low words
ZB_DEVINL void mma_ss(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "mov.b64 da, {%1, %5};\n\t"
        "mov.b64 db, {%2, %5};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(DESC_HI)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], B's descriptor given by its low word
ZB_DEVINL void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "mov.b64 db, {%2, %5};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(DESC_HI)
        : "memory");
}

// The key tile of step j of an item: selected tile idx[j] (clamped), or -1 for a landmark chunk.
ZB_DEVINL int step_tile(const Params& p, const int32_t* list, int j) {
    if (j >= p.k) return -1;
    if (p.dense) return j;
    int t = __ldg(list + j);
    return t < 0 ? 0 : (t >= p.Tk ? p.Tk - 1 : t);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kb,
                   const __grid_constant__ CUtensorMap tm_vb, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = warp_id();
    const int lane = lane_id();
    const int wg = warp >> 2;
    const WaitCtx wc{p.status, &sm.abort_flag, p.timeout_ns};
    const int n = p.k + p.lm_chunks;  // steps per item
    const long long first = blockIdx.x, G = gridDim.x;
    const int cnt = first < p.n_items ? static_cast<int>((p.n_items - 1 - first) / G + 1) : 0;
    const int rounds = (cnt + 1) / 2;

    // ---------------------------------------------------------- set-up ----
    // Zero the operand buffers once: a 64-row TMA box leaves rows 64..127 of
    // a buffer untouched, and those rows must hold finite values.
    {
        uint4* z = reinterpret_cast<uint4*>(&sm.q[0][0]);
        const int n16 = (SLOTS + K_STAGES + V_STAGES) * TILE_BYTES / 16;
        for (int i = threadIdx.x; i < n16; i += NUM_THREADS) z[i] = make_uint4(0, 0, 0, 0);
    }
    if (threadIdx.x == 0) {
        sm.abort_flag = 0;
        for (int s = 0; s < SLOTS; ++s) {
            mbar_init(smem_addr(&sm.q_full[s]), 1);
            mbar_init(smem_addr(&sm.q_empty[s]), 1);
            mbar_init(smem_addr(&sm.s_full[s]), 1);
            mbar_init(smem_addr(&sm.s_free[s]), 128);
            mbar_init(smem_addr(&sm.p_full[s]), 128);
            mbar_init(smem_addr(&sm.p_free[s]), 1);
            mbar_init(smem_addr(&sm.o_free[s]), 128);
        }
        for (int i = 0; i < K_STAGES; ++i) {
            mbar_init(smem_addr(&sm.k_full[i]), 1);
            mbar_init(smem_addr(&sm.k_empty[i]), 1);
        }
        for (int i = 0; i < V_STAGES; ++i) {
            mbar_init(smem_addr(&sm.v_full[i]), 1);
            mbar_init(smem_addr(&sm.v_empty[i]), 1);
        }
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

    if (warp == 0 || warp == 2) {
        if (lane == 0) {
            // =========================== producers: warp 0 Q + K, warp 2 V ====
            const bool is_k = warp == 0;
            const int STAGES = is_k ? K_STAGES : V_STAGES;
            uint64_t* full = is_k ? sm.k_full : sm.v_full;
            uint64_t* empty = is_k ? sm.k_empty : sm.v_empty;
            uint8_t(*buf)[TILE_BYTES] = is_k ? sm.k : sm.v;
            const CUtensorMap* map = is_k ? &tm_k : &tm_v;
            const CUtensorMap* lmap = is_k ? &tm_kb : &tm_vb;
            uint32_t seq = 0;                    // loads issued into the ring
            uint32_t issued_mask = 0, parity_mask = 0, q_issued = 0, q_parity = 0;
            bool ok = true;
            for (int r = 0; r < rounds && ok; ++r) {
                const int A = (2 * r + 1 < cnt) ? 2 : 1;
                int hs[SLOTS], is_[SLOTS];
                const int32_t* lists[SLOTS];
#pragma unroll
                for (int s = 0; s < SLOTS; ++s) {
                    if (s >= A) break;
                    const long long item = first + static_cast<long long>(2 * r + s) * G;
                    hs[s] = static_cast<int>(item / p.Tq);
                    is_[s] = static_cast<int>(item % p.Tq);
                    lists[s] = p.dense ? nullptr : p.idx + item * static_cast<long long>(p.k);
                    if (is_k) {
                        if (!mbar_wait(smem_addr(&sm.q_empty[s]), (r & 1) ^ 1, wc)) { ok = false; break; }
                        const uint32_t bar = smem_addr(&sm.q_full[s]);
                        mbar_arrive_expect_tx(bar, p.tq * HD * 2);
                        tma_load_3d(smem_addr(sm.q[s]), &tm_q, bar, 0, is_[s] * p.tq, hs[s]);
                        q_issued |= 1u << s;
                        q_parity = (q_parity & ~(1u << s)) | ((r & 1u) << s);
                    }
                }
                if (!ok) break;
                for (int j = 0; j < n && ok; ++j) {
#pragma unroll
                    for (int s = 0; s < SLOTS; ++s) {
                        if (s >= A) break;
                        const int st = static_cast<int>(seq % STAGES);
                        const uint32_t use = seq / STAGES;
                        if (!mbar_wait(smem_addr(&empty[st]), (use & 1) ^ 1, wc)) { ok = false; break; }
                        const uint32_t bar = smem_addr(&full[st]);
                        const int t = step_tile(p, lists[s], j);
                        if (t >= 0) {
                            mbar_arrive_expect_tx(bar, p.tk * HD * 2);
                            tma_load_3d(smem_addr(buf[st]), map, bar, 0, t * p.tk, hs[s]);
                        } else {
                            mbar_arrive_expect_tx(bar, TILE_BYTES);
                            tma_load_3d(smem_addr(buf[st]), lmap, bar, 0, (j - p.k) * BN, hs[s]);
                        }
                        issued_mask |= 1u << st;
                        parity_mask = (parity_mask & ~(1u << st)) | ((use & 1u) << st);
                        ++seq;
                    }
                }
            }
            // leave no TMA write in flight (bounded, even after an abort)
            volatile int no_abort = 0;
            const WaitCtx w2{p.status, &no_abort, p.timeout_ns};
            for (int st = 0; st < STAGES; ++st)
                if ((issued_mask >> st) & 1u) mbar_wait(smem_addr(&full[st]), (parity_mask >> st) & 1u, w2);
            for (int s = 0; s < SLOTS; ++s)
                if ((q_issued >> s) & 1u) mbar_wait(smem_addr(&sm.q_full[s]), (q_parity >> s) & 1u, w2);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================================================= MMA issuer ====
        constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, 0, 0);  // Q K-major, K K-major
        constexpr uint32_t IDESC_PV = idesc_bf16(BM, HD, 0, 1);  // P (TMEM), V MN-major
        if (lane == 0) {
            const uint32_t q_lo0 = desc_lo(smem_addr(sm.q[0]), 16);
            const uint32_t k_lo0 = desc_lo(smem_addr(sm.k[0]), 16);
            const uint32_t v_lo0 = desc_lo(smem_addr(sm.v[0]), 0);
            constexpr uint32_t TILE_LO = TILE_BYTES >> 4;
            int k_next = 0, v_next = 0;
            uint32_t k_ph = 0, v_ph = 0;
            bool ok = true;
            auto issue_qk = [&](int s, long long g) -> bool {
                const int ks = k_next;
                if (!mbar_wait_sleep(smem_addr(&sm.k_full[ks]), k_ph, wc, SLEEP_NS)) return false;
                if (++k_next == K_STAGES) { k_next = 0; k_ph ^= 1u; }
                if (!mbar_wait_sleep(smem_addr(&sm.s_free[s]), static_cast<uint32_t>((g & 1) ^ 1), wc, SLEEP_NS)) return false;
                tc_fence_after();
                const uint32_t qa = q_lo0 + s * TILE_LO, kb = k_lo0 + ks * TILE_LO;
                const uint32_t d_tmem = tmem + s * SLOT_COLS + TM_S;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) mma_ss(d_tmem, qa + kk * 2, kb + kk * 2, IDESC_QK, kk > 0 ? 1u : 0u);
                umma_commit(smem_addr(&sm.s_full[s]));
                umma_commit(smem_addr(&sm.k_empty[ks]));
                return true;
            };
            for (int r = 0; r < rounds && ok; ++r) {
                const int A = (2 * r + 1 < cnt) ? 2 : 1;
                for (int s = 0; s < A && ok; ++s)
                    if (!mbar_wait_sleep(smem_addr(&sm.q_full[s]), r & 1, wc, SLEEP_NS)) ok = false;
                if (!ok) break;
                tc_fence_after();
                for (int s = 0; s < A && ok; ++s)
                    if (!issue_qk(s, static_cast<long long>(r) * n)) ok = false;
                for (int j = 0; j < n && ok; ++j) {
                    for (int s = 0; s < A; ++s) {
                        const long long g = static_cast<long long>(r) * n + j;
                        if (j + 1 < n) {
                            if (!issue_qk(s, g + 1)) { ok = false; break; }
                        } else {
                            umma_commit(smem_addr(&sm.q_empty[s]));
                        }
                        if (!mbar_wait_sleep(smem_addr(&sm.p_full[s]), static_cast<uint32_t>(g & 1), wc, SLEEP_NS)) { ok = false; break; }
                        if (j == 0) {
                            if (!mbar_wait_sleep(smem_addr(&sm.o_free[s]), (r & 1) ^ 1, wc, SLEEP_NS)) { ok = false; break; }
                        }
                        const int vs = v_next;
                        if (!mbar_wait_sleep(smem_addr(&sm.v_full[vs]), v_ph, wc, SLEEP_NS)) { ok = false; break; }
                        if (++v_next == V_STAGES) { v_next = 0; v_ph ^= 1u; }
                        tc_fence_after();
                        const uint32_t vb = v_lo0 + vs * TILE_LO;
                        const uint32_t p_tmem = tmem + s * SLOT_COLS + TM_P;
                        const uint32_t o_tmem = tmem + s * SLOT_COLS + TM_O;
#pragma unroll
                        for (int kk = 0; kk < BN / 16; ++kk)
                            mma_ts(o_tmem, p_tmem + kk * 8, vb + kk * 128, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(smem_addr(&sm.v_empty[vs]));
                        umma_commit(smem_addr(&sm.p_free[s]));
                    }
                }
            }
            // no tcgen05.mma may still run when TMEM is released
            umma_commit(smem_addr(&sm.drain));
            volatile int no_abort = 0;
            const WaitCtx w2{p.status, &no_abort, p.timeout_ns};
            mbar_wait(smem_addr(&sm.drain), 0, w2);
        }
        __syncwarp();
    } else if (warp == 3) {
        // ============================ index-list check (off the critical path) ====
        // Every list must be in range and strictly ascending; a bad one sets
        // ZB_ERR_INDEX (the kernel itself clamps indices and never reads out of
        // bounds).  32 entries per step, one per lane.
        if (!p.dense) {
            for (int it = 0; it < cnt; ++it) {
                const long long item = first + static_cast<long long>(it) * G;
                const int32_t* list = p.idx + item * static_cast<long long>(p.k);
                int bad = 0;
                for (int q0 = 0; q0 < p.k; q0 += 32) {
                    const int q = q0 + lane;
                    const int t = q < p.k ? __ldg(list + q) : 0;
                    int prev = __shfl_up_sync(0xffffffffu, t, 1);
                    if (lane == 0) prev = q0 == 0 ? -1 : __ldg(list + q0 - 1);
                    if (q < p.k && (t < 0 || t >= p.Tk || t <= prev)) bad = 1;
                }
                if (__any_sync(0xffffffffu, bad)) {
                    if (lane == 0) flag_status(p.status, ZB_ERR_INDEX);
                    break;
                }
            }
        }
    } else if (wg >= 1) {
        // ===================================== softmax warpgroup of a slot ====
        const int s = wg - 1;
        const int quarter = warp & 3;            // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;     // query row within the tile
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tm_s = tmem + lane_addr + s * SLOT_COLS + TM_S;
        const uint32_t tm_p = tmem + lane_addr + s * SLOT_COLS + TM_P;
        const uint32_t tm_o = tmem + lane_addr + s * SLOT_COLS + TM_O;
        bool ok = true;
        for (int r = 0; r < rounds && ok; ++r) {
            const int it = 2 * r + s;
            if (it >= cnt) break;
            const long long item = first + static_cast<long long>(it) * G;
            const int h = static_cast<int>(item / p.Tq);
            const int i = static_cast<int>(item % p.Tq);
            const int32_t* list = p.dense ? nullptr : p.idx + item * static_cast<long long>(p.k);
            // valid columns of the last selected tile (only the last key tile is ragged)
            int last_valid = p.tk;
            if (p.k > 0) {
                const int jl = p.dense ? p.Tk - 1 : __ldg(list + p.k - 1);
                if (jl == p.Tk - 1) last_valid = p.n_last;
            }
            int ip = 0;           // walk over the sorted index list for landmark masks
            float m = -INFINITY;  // running max of the log2-domain logits (lazy)
            float l = 0.f;        // running sum of 2^(x - m)
            long long g = static_cast<long long>(r) * n;
            for (int j = 0; j < n; ++j, ++g) {
                if (!mbar_wait(smem_addr(&sm.s_full[s]), static_cast<uint32_t>(g & 1), wc)) { ok = false; break; }
                tc_fence_after();
                const bool is_lm = j >= p.k;
                // Per-column treatment of S: selected tiles mask columns past the
                // tile's length; landmark chunks become s * scale + log2(n_j), or
                // -inf for selected / out-of-range tiles (the selected ones come
                // from a walk over the sorted index list, kept in 4 mask words).
                const int valid = is_lm ? BN : ((j == p.k - 1) ? last_valid : p.tk);
                const int j0 = (j - p.k) * BN;
                uint32_t s0 = 0u, s1 = 0u, s2 = 0u, s3 = 0u;
                if (is_lm) {
                    while (ip < p.k) {
                        const int t = __ldg(list + ip);
                        if (t >= j0 + BN) break;
                        if (t >= j0) {
                            const int c = t - j0;
                            const uint32_t bit = 1u << (c & 31);
                            s0 |= (c >> 5) == 0 ? bit : 0u;
                            s1 |= (c >> 5) == 1 ? bit : 0u;
                            s2 |= (c >> 5) == 2 ? bit : 0u;
                            s3 |= (c >> 5) == 3 ? bit : 0u;
                        }
                        ++ip;
                    }
                    const int past = p.Tk - j0;  // columns >= past are beyond the last tile
                    if (past < 32) s0 |= past <= 0 ? 0xFFFFFFFFu : (0xFFFFFFFFu << past);
                    if (past < 64) s1 |= past <= 32 ? 0xFFFFFFFFu : (0xFFFFFFFFu << (past - 32));
                    if (past < 96) s2 |= past <= 64 ? 0xFFFFFFFFu : (0xFFFFFFFFu << (past - 64));
                    if (past < 128) s3 |= past <= 96 ? 0xFFFFFFFFu : (0xFFFFFFFFu << (past - 96));
                }
                // Per-column treatment of chunk c of S (raw words r): selected tiles
                // mask columns past the tile's length; landmark chunks become
                // s * scale + log2(n_j), or -inf for selected / out-of-range tiles.
                auto treat = [&](float (&y)[32], const uint32_t (&r)[32], int c) {
                    if (is_lm) {
                        const uint32_t bits = c == 0 ? s0 : (c == 1 ? s1 : (c == 2 ? s2 : s3));
                        const int lastc = p.Tk - 1 - j0 - c * 32;  // column of the ragged last tile
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            float bias = (e == lastc) ? p.log2_last : p.log2_tk;
                            if ((bits >> e) & 1u) bias = -INFINITY;
                            y[e] = fmaf(__uint_as_float(r[e]), p.scale_log2, bias);
                        }
                    } else {
                        const int vc = valid - c * 32;  // valid columns in this chunk
#pragma unroll
                        for (int e = 0; e < 32; ++e) y[e] = __uint_as_float(r[e]);
                        if (vc < 32) {  // only a ragged last tile (or a 64-row tile) needs the mask
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (e >= vc) y[e] = -INFINITY;
                        }
                    }
                };
                // one 32-column chunk c of S into y[] (treated)
                auto load_chunk = [&](float (&y)[32], int c) {
                    uint32_t r[32];
                    tmem_ld32(tm_s + c * 32, r);
                    tmem_wait_ld_dep(r);
                    treat(y, r, c);
                };
                // chunks c and c + 1 with one TMEM wait
                auto load_chunk2 = [&](float (&y)[32], float (&z)[32], int c) {
                    uint32_t r[32], r2[32];
                    tmem_ld32(tm_s + c * 32, r);
                    tmem_ld32(tm_s + c * 32 + 32, r2);
                    tmem_wait_ld_dep(r);
                    tmem_wait_ld_dep(r2);
                    treat(y, r, c);
                    treat(z, r2, c + 1);
                };
                // ---- pass 1: row max (two chunks per TMEM wait)
                float mx = -INFINITY;
#pragma unroll 1
                for (int c = 0; c < BN / 32; c += 2) {
                    float y[32], z[32];
                    load_chunk2(y, z, c);
                    float g0 = fmax3(y[0], y[1], y[2]), g1 = fmax3(z[0], z[1], z[2]);
                    float g2 = fmax3(y[3], y[4], y[5]), g3 = fmax3(z[3], z[4], z[5]);
#pragma unroll
                    for (int e = 6; e < 30; e += 2) {
                        g0 = fmax3(g0, y[e], y[e + 1]);
                        g1 = fmax3(g1, z[e], z[e + 1]);
                    }
                    g2 = fmax3(g2, y[30], y[31]);
                    g3 = fmax3(g3, z[30], z[31]);
                    mx = fmaxf(mx, fmaxf(fmax3(g0, g1, g2), g3));
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
                const float nm = (m == -INFINITY) ? 0.f : -m;
                const float cm = is_lm ? 1.f : p.scale_log2;  // landmark logits are already scaled
                // P of this slot is free once P V of the previous step is done;
                // O then holds every earlier step and can be rescaled
                if (!mbar_wait(smem_addr(&sm.p_free[s]), static_cast<uint32_t>((g & 1) ^ 1), wc)) { ok = false; break; }
                tc_fence_after();
                if (rescale && j > 0) {
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t ro[32];
                        tmem_ld32(tm_o + c * 32, ro);
                        tmem_wait_ld_dep(ro);
#pragma unroll
                        for (int e = 0; e < 32; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * alpha);
                        tmem_st32(tm_o + c * 32, ro);
                        tmem_wait_st();
                    }
                }
                // ---- pass 2: p = 2^(x * cm - m) per chunk (1 of 4 pairs on the FMA
                // pipes, the rest on MUFU), packed fp32x2, bf16 pairs straight to TMEM
                const uint64_t cm2 = f2_pack(cm, cm), nm2 = f2_pack(nm, nm);
                uint64_t acc0 = 0ull, acc1 = 0ull;
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    float y[32];
                    load_chunk(y, c);
                    if (c == BN / 32 - 1) {
                        tc_fence_before();
                        mbar_arrive(smem_addr(&sm.s_free[s]));  // S fully read: the next Q K^T may overwrite it
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const uint64_t xs = f2_fma(f2_pack(y[2 * q], y[2 * q + 1]), cm2, nm2);
                        uint64_t pv;
                        if ((q & 3) == 1) {
                            pv = f2_exp2_poly(xs);
                        } else {
                            float a0, a1;
                            f2_unpack(xs, a0, a1);
                            pv = f2_pack(ex2(a0), ex2(a1));
                        }
                        if (q & 1) acc1 = f2_add(acc1, pv); else acc0 = f2_add(acc0, pv);
                        float p0, p1;
                        f2_unpack(pv, p0, p1);
                        pk[q] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(tm_p + c * 16, pk);
                }
                float rs0, rs1;
                f2_unpack(f2_add(acc0, acc1), rs0, rs1);
                l += rs0 + rs1;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_addr(&sm.p_full[s]));
            }
            if (!ok) break;
            // ------------------------------------------------ epilogue ----
            const long long gl = g - 1;
            if (!mbar_wait(smem_addr(&sm.p_free[s]), static_cast<uint32_t>(gl & 1), wc)) { ok = false; break; }
            tc_fence_after();
            float o[HD];
            {
                uint32_t ro[HD];
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) tmem_ld32(tm_o + c * 32, sub32(ro, c * 32));
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) tmem_wait_ld_dep(sub32(ro, c * 32));
#pragma unroll
                for (int e = 0; e < HD; ++e) o[e] = __uint_as_float(ro[e]);
            }
            tc_fence_before();
            mbar_arrive(smem_addr(&sm.o_free[s]));
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
