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
// per 128 x 128 tile) costs more than the tile's two MMAs, so two softmax
// warpgroups run at the same time, and each slot is a pipeline of its own
// (producer, MMA issuer, softmax) that shares nothing with the other slot but
// the SM.
//   warps 0 / 2  producer of slot 0 / 1 (one lane, TMA): Q of each item, then
//                per step the K and V tile of the selected key tile or
//                landmark chunk, K and V each in a ring of their own.
//   warps 1 / 3  MMA issuer of slot 0 / 1 (one lane): S = Q K^T into the
//                slot's TMEM S as soon as the softmax has read the previous S,
//                then O += P V with P read from TMEM (tcgen05 "TS" form).
//   warps 4..7   softmax of slot 0, warps 8..11 softmax of slot 1: one thread
//                per query row reads its whole S row into registers (S is then
//                free for the next Q K^T), log2-domain online softmax with
//                lazy rescaling of O, P (bf16) to TMEM, epilogue O / l.  They
//                also check the index lists and keep the slot's bitmap of
//                selected tiles from which the landmark masks are read.
// Items are dealt round-robin over CTAs, so CTAs running at the same time work
// on neighbouring query tiles of one head and sweep its K/V in ascending order
// together (L2 reuse).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <type_traits>

#include "zb_common.cuh"
#include "zb_host.h"

namespace zb {
namespace attn {

constexpr int BM = 128;          // query rows per work item (MMA M)
constexpr int BN = 128;          // keys per step (QK MMA N, PV MMA K)
constexpr int HD = 64;           // head dim
constexpr int SLOTS = 2;
constexpr int K_STAGES = 3;      // per slot
constexpr int V_STAGES = 2;      // per slot
constexpr int NUM_THREADS = 384;
constexpr int MAX_TILES = 32768;
constexpr uint32_t TILE_BYTES = BN * HD * 2;  // 16 KB, one 128 x 64 bf16 tile
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns of slot s start at 256 s: S (128 fp32), P (64 = 128 bf16), O (64 fp32)
constexpr uint32_t SLOT_COLS = 256, TM_S = 0, TM_P = 128, TM_O = 192;
constexpr uint32_t SLEEP_NS = 20000;  // longest sleep inside one barrier poll of a role thread
// Registers: the kernel is compiled for LAUNCH_REGS per thread (384 threads,
// one CTA per SM); the role warpgroup then gives registers back and the two
// softmax warpgroups take them (setmaxnreg), which adds up exactly:
// 128 * ROLE_REGS + 256 * SOFTMAX_REGS == 384 * LAUNCH_REGS.
constexpr int LAUNCH_REGS = 168, ROLE_REGS = 56, SOFTMAX_REGS = 224;
static_assert(128 * ROLE_REGS + 256 * SOFTMAX_REGS == NUM_THREADS * LAUNCH_REGS, "register split");

constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: p <= 2^8 before a rescale

// Everything of one slot's pipeline: its operand tiles (1024-byte aligned, as
// the 128-byte swizzle needs) and barriers.
struct __align__(1024) SlotSmem {
    uint8_t q[TILE_BYTES];
    uint8_t k[K_STAGES][TILE_BYTES];
    uint8_t v[V_STAGES][TILE_BYTES];
    uint64_t q_full, q_empty;
    uint64_t k_full[K_STAGES], k_empty[K_STAGES];
    uint64_t v_full[V_STAGES], v_empty[V_STAGES];
    uint64_t s_full, s_free, p_full, p_free, o_free;
    uint64_t drain;
};

struct Smem {
    SlotSmem slot[SLOTS];
    // Selected key tiles of each slot's current and next item as bitmaps (for
    // the landmark masks); built at the item's start, cleared after its last P V.
    uint32_t bm[SLOTS][2][MAX_TILES / 32];
    uint64_t bm_ready[SLOTS][2];
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
    unsigned* wave;    // zeroed counter for the wave synchronisation, or NULL
    int* status;
    unsigned long long timeout_ns;
};

template <int N>
ZB_DEVINL void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N>
ZB_DEVINL void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }

// 32 lanes x 16 consecutive 32-bit columns
ZB_DEVINL void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
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

// Wave synchronisation across the grid: spin (bounded) until *ctr >= target.
ZB_DEVINL bool wave_wait(const unsigned* ctr, unsigned target, const WaitCtx& w) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= target) return true;
        if ((it & 15u) == 15u) {
            if (*w.abort_flag) return false;
            if (globaltimer_ns() - t0 > w.timeout_ns) {
                flag_status(w.status, ZB_ERR_TIMEOUT);
                *w.abort_flag = 1;
                return false;
            }
        }
        __nanosleep(128);
    }
}

// The key tile of step j of an item: selected tile idx[j] (clamped), or -1 for a landmark chunk.
ZB_DEVINL int step_tile(const Params& p, const int32_t* list, int j) {
    if (j >= p.k) return -1;
    if (p.dense) return j;
    int t = __ldg(list + j);
    return t < 0 ? 0 : (t >= p.Tk ? p.Tk - 1 : t);
}

// LM: whether the launch has landmark chunks.  The launches without (dense
// attention, tile-sparse without landmarks) use an instantiation that holds no
// landmark code at all, which keeps their step loop short.
template <bool LM>
__global__ void __launch_bounds__(NUM_THREADS, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kb,
                   const __grid_constant__ CUtensorMap tm_vb, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = warp_id();
    const int lane = lane_id();
    const WaitCtx wc{p.status, &sm.abort_flag, p.timeout_ns};
    const int n = p.k + p.lm_chunks;  // steps per item
    const long long first = blockIdx.x, G = gridDim.x;
    const int cnt = first < p.n_items ? static_cast<int>((p.n_items - 1 - first) / G + 1) : 0;

    // ---------------------------------------------------------- set-up ----
    // Zero the operand tiles once: a 64-row TMA box leaves rows 64..127 of a
    // tile untouched, and those rows must hold finite values.
    for (int s = 0; s < SLOTS; ++s) {
        uint4* z = reinterpret_cast<uint4*>(sm.slot[s].q);
        const int n16 = (1 + K_STAGES + V_STAGES) * TILE_BYTES / 16;
        for (int i = threadIdx.x; i < n16; i += NUM_THREADS) z[i] = make_uint4(0, 0, 0, 0);
    }
    if (p.lm_chunks) {
        uint32_t* z = &sm.bm[0][0][0];
        for (int i = threadIdx.x; i < SLOTS * 2 * (MAX_TILES / 32); i += NUM_THREADS) z[i] = 0u;
    }
    if (threadIdx.x == 0) {
        sm.abort_flag = 0;
        for (int s = 0; s < SLOTS; ++s) {
            mbar_init(smem_addr(&sm.bm_ready[s][0]), 128);
            mbar_init(smem_addr(&sm.bm_ready[s][1]), 128);
        }
        for (int s = 0; s < SLOTS; ++s) {
            SlotSmem& b = sm.slot[s];
            mbar_init(smem_addr(&b.q_full), 1);
            mbar_init(smem_addr(&b.q_empty), 1);
            for (int i = 0; i < K_STAGES; ++i) {
                mbar_init(smem_addr(&b.k_full[i]), 1);
                mbar_init(smem_addr(&b.k_empty[i]), 1);
            }
            for (int i = 0; i < V_STAGES; ++i) {
                mbar_init(smem_addr(&b.v_full[i]), 1);
                mbar_init(smem_addr(&b.v_empty[i]), 1);
            }
            mbar_init(smem_addr(&b.s_full), 1);
            mbar_init(smem_addr(&b.s_free), 128);
            mbar_init(smem_addr(&b.p_full), 128);
            mbar_init(smem_addr(&b.p_free), 1);
            mbar_init(smem_addr(&b.o_free), 128);
            mbar_init(smem_addr(&b.drain), 1);
        }
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

    if (warp < 4) {
        setmaxnreg_dec<ROLE_REGS>();
        // Role warps: warp 0 / 2 produce for slot 0 / 1, warp 1 / 3 issue its
        // MMAs.  The two slots' pipelines share nothing but the SM.
        const int s = warp >> 1;
        SlotSmem& b = sm.slot[s];
        const int items = (cnt + 1 - s) / 2;  // this slot's items: it = 2 r + s
        if ((warp & 1) == 0 && lane == 0) {
            // ================================================ producer ====
            // Q of each item, then per step the K and V tile of the selected
            // key tile or landmark chunk, each into its own ring.
            int kst = 0, vst = 0;
            uint32_t kph = 0, vph = 0;
            uint32_t k_issued = 0, v_issued = 0, k_par = 0, v_par = 0;
            bool q_issued = false;
            uint32_t q_par = 0;
            bool ok = true;
            // Wave synchronisation (when the caller passed a counter): round r
            // starts on both slots of every CTA together, so the items in
            // flight sweep the head's K/V in step and share it through L2.
            // Barrier r >= 1 is passed when all 2 G producers have arrived; R
            // rounds in all (the most any slot of any CTA has).
            const int R = (static_cast<int>((p.n_items - 1) / G) + 2) / 2;
            int arrived = 0;  // barriers arrived at so far
            for (int r = 0; r < items && ok; ++r) {
                if (p.wave && r >= 1) {
                    atomicAdd(p.wave, 1u);
                    arrived = r;
                    if (!wave_wait(p.wave, static_cast<unsigned>(r) * 2u * static_cast<unsigned>(G), wc)) break;
                }
                const long long item = first + static_cast<long long>(2 * r + s) * G;
                const int h = static_cast<int>(item / p.Tq);
                const int i = static_cast<int>(item % p.Tq);
                const int32_t* list = p.dense ? nullptr : p.idx + item * static_cast<long long>(p.k);
                if (!mbar_wait_sleep(smem_addr(&b.q_empty), (r & 1) ^ 1, wc, SLEEP_NS)) break;
                mbar_arrive_expect_tx(smem_addr(&b.q_full), p.tq * HD * 2);
                tma_load_3d(smem_addr(b.q), &tm_q, smem_addr(&b.q_full), 0, i * p.tq, h);
                q_issued = true;
                q_par = r & 1u;
                // K and V fill their rings independently (K leads: S = Q K^T
                // of a step is needed before its P V), so a slow V stage never
                // holds back the K loads.  Non-blocking tests; after a round
                // without progress a short sleep, and a time limit.
                int kj = 0, vj = 0;  // next K / V step of the item to load
                uint64_t idle_since = 0;
                while (vj < n) {
                    bool progressed = false;
                    if (kj < n && mbar_test(smem_addr(&b.k_empty[kst]), kph ^ 1u)) {
                        const int t = step_tile(p, list, kj);
                        if (t >= 0) {
                            mbar_arrive_expect_tx(smem_addr(&b.k_full[kst]), p.tk * HD * 2);
                            tma_load_3d(smem_addr(b.k[kst]), &tm_k, smem_addr(&b.k_full[kst]), 0, t * p.tk, h);
                        } else {
                            mbar_arrive_expect_tx(smem_addr(&b.k_full[kst]), TILE_BYTES);
                            tma_load_3d(smem_addr(b.k[kst]), &tm_kb, smem_addr(&b.k_full[kst]), 0, (kj - p.k) * BN, h);
                        }
                        k_issued |= 1u << kst;
                        k_par = (k_par & ~(1u << kst)) | (kph << kst);
                        if (++kst == K_STAGES) { kst = 0; kph ^= 1u; }
                        ++kj;
                        progressed = true;
                    }
                    if (vj < kj && mbar_test(smem_addr(&b.v_empty[vst]), vph ^ 1u)) {
                        const int t = step_tile(p, list, vj);
                        if (t >= 0) {
                            mbar_arrive_expect_tx(smem_addr(&b.v_full[vst]), p.tk * HD * 2);
                            tma_load_3d(smem_addr(b.v[vst]), &tm_v, smem_addr(&b.v_full[vst]), 0, t * p.tk, h);
                        } else {
                            mbar_arrive_expect_tx(smem_addr(&b.v_full[vst]), TILE_BYTES);
                            tma_load_3d(smem_addr(b.v[vst]), &tm_vb, smem_addr(&b.v_full[vst]), 0, (vj - p.k) * BN, h);
                        }
                        v_issued |= 1u << vst;
                        v_par = (v_par & ~(1u << vst)) | (vph << vst);
                        if (++vst == V_STAGES) { vst = 0; vph ^= 1u; }
                        ++vj;
                        progressed = true;
                    }
                    if (progressed) {
                        idle_since = 0;
                        continue;
                    }
                    const uint64_t now = globaltimer_ns();
                    if (idle_since == 0) idle_since = now;
                    if (*wc.abort_flag) { ok = false; break; }
                    if (now - idle_since > p.timeout_ns) {
                        flag_status(p.status, ZB_ERR_TIMEOUT);
                        *wc.abort_flag = 1;
                        ok = false;
                        break;
                    }
                    __nanosleep(64);
                }
            }
            // arrive at the barriers of the rounds this CTA does not run (so the
            // others pass them), then leave no TMA write in flight (bounded,
            // even after an abort)
            if (p.wave)
                for (int r = arrived + 1; r < R; ++r) atomicAdd(p.wave, 1u);
            volatile int no_abort = 0;
            const WaitCtx w2{p.status, &no_abort, drain_timeout_ns(p.timeout_ns)};
            for (int st = 0; st < K_STAGES; ++st)
                if ((k_issued >> st) & 1u) mbar_wait(smem_addr(&b.k_full[st]), (k_par >> st) & 1u, w2);
            for (int st = 0; st < V_STAGES; ++st)
                if ((v_issued >> st) & 1u) mbar_wait(smem_addr(&b.v_full[st]), (v_par >> st) & 1u, w2);
            if (q_issued) mbar_wait(smem_addr(&b.q_full), q_par, w2);
        } else if ((warp & 1) == 1 && lane == 0) {
            // ============================================== MMA issuer ====
            // Per step: S = Q K^T (as soon as the softmax has read the previous
            // S), then O += P V with P read from TMEM (tcgen05 "TS" form).
            constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, 0, 0);  // Q K-major, K K-major
            constexpr uint32_t IDESC_PV = idesc_bf16(BM, HD, 0, 1);  // P (TMEM), V MN-major
            const uint32_t q_lo = desc_lo(smem_addr(b.q), 16);
            const uint32_t k_lo0 = desc_lo(smem_addr(b.k[0]), 16);
            const uint32_t v_lo0 = desc_lo(smem_addr(b.v[0]), 0);
            constexpr uint32_t TILE_LO = TILE_BYTES >> 4;
            const uint32_t s_tmem = tmem + s * SLOT_COLS + TM_S;
            const uint32_t p_tmem = tmem + s * SLOT_COLS + TM_P;
            const uint32_t o_tmem = tmem + s * SLOT_COLS + TM_O;
            int kst = 0, vst = 0;
            uint32_t kph = 0, vph = 0;
            long long g = 0;  // steps of this slot so far
            bool ok = true;
            auto issue_qk = [&]() -> bool {
                if (!mbar_wait_sleep(smem_addr(&b.k_full[kst]), kph, wc, SLEEP_NS)) return false;
                if (!mbar_wait_sleep(smem_addr(&b.s_free), static_cast<uint32_t>((g & 1) ^ 1), wc, SLEEP_NS)) return false;
                tc_fence_after();
                const uint32_t kb = k_lo0 + kst * TILE_LO;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) mma_ss(s_tmem, q_lo + kk * 2, kb + kk * 2, IDESC_QK, kk > 0 ? 1u : 0u);
                umma_commit(smem_addr(&b.s_full));
                umma_commit(smem_addr(&b.k_empty[kst]));
                if (++kst == K_STAGES) { kst = 0; kph ^= 1u; }
                return true;
            };
            for (int r = 0; r < items && ok; ++r) {
                if (!mbar_wait_sleep(smem_addr(&b.q_full), r & 1, wc, SLEEP_NS)) break;
                tc_fence_after();
                if (!issue_qk()) break;  // S of step 0 (g is its step number)
                for (int j = 0; j < n; ++j, ++g) {
                    if (j + 1 < n) {
                        ++g;
                        const bool q_ok = issue_qk();
                        --g;
                        if (!q_ok) { ok = false; break; }
                    } else {
                        umma_commit(smem_addr(&b.q_empty));
                    }
                    if (!mbar_wait_sleep(smem_addr(&b.p_full), static_cast<uint32_t>(g & 1), wc, SLEEP_NS)) { ok = false; break; }
                    if (j == 0) {
                        if (!mbar_wait_sleep(smem_addr(&b.o_free), (r & 1) ^ 1, wc, SLEEP_NS)) { ok = false; break; }
                    }
                    if (!mbar_wait_sleep(smem_addr(&b.v_full[vst]), vph, wc, SLEEP_NS)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t vb = v_lo0 + vst * TILE_LO;
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        mma_ts(o_tmem, p_tmem + kk * 8, vb + kk * 128, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(smem_addr(&b.v_empty[vst]));
                    umma_commit(smem_addr(&b.p_free));
                    if (++vst == V_STAGES) { vst = 0; vph ^= 1u; }
                }
            }
            // no tcgen05.mma of this thread may still run when TMEM is released
            umma_commit(smem_addr(&b.drain));
            volatile int no_abort = 0;
            const WaitCtx w2{p.status, &no_abort, drain_timeout_ns(p.timeout_ns)};
            mbar_wait(smem_addr(&b.drain), 0, w2);
        }
        __syncwarp();
    } else {
        setmaxnreg_inc<SOFTMAX_REGS>();
        // ===================================== softmax warpgroup of a slot ====
        const int s = (warp >> 2) - 1;
        SlotSmem& b = sm.slot[s];
        const int quarter = warp & 3;            // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;     // query row within the tile
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tm_s = tmem + lane_addr + s * SLOT_COLS + TM_S;
        const uint32_t tm_p = tmem + lane_addr + s * SLOT_COLS + TM_P;
        const uint32_t tm_o = tmem + lane_addr + s * SLOT_COLS + TM_O;
        const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
        const int items = (cnt + 1 - s) / 2;
        uint32_t ph = 0;  // parity of this slot's step counter
        bool ok = true;
        for (int r = 0; r < items && ok; ++r) {
            const long long item = first + static_cast<long long>(2 * r + s) * G;
            const int h = static_cast<int>(item / p.Tq);
            const int i = static_cast<int>(item % p.Tq);
            const int32_t* list = p.dense ? nullptr : p.idx + item * static_cast<long long>(p.k);
            // Index-list check, 1/128 of the list per thread: in range and
            // strictly ascending, else ZB_ERR_INDEX (the producers clamp, so a
            // bad list never leads to an out-of-bounds read).
            // With landmarks, the same pass marks the selected tiles in this
            // item's bitmap (indices clamped into range).
            uint32_t* bm = sm.bm[s][r & 1];
            if (list) {
                int bad = 0;
                for (int q = row; q < p.k; q += BM) {
                    const int t = __ldg(list + q);
                    const int prev = q > 0 ? __ldg(list + q - 1) : -1;
                    bad |= (t < 0) | (t >= p.Tk) | (t <= prev);
                    if (p.lm_chunks) {
                        const int tc = t < 0 ? 0 : (t >= p.Tk ? p.Tk - 1 : t);
                        atomicOr(&bm[tc >> 5], 1u << (tc & 31));
                    }
                }
                if (bad) flag_status(p.status, ZB_ERR_INDEX);
            }
            if (p.lm_chunks) mbar_arrive(smem_addr(&sm.bm_ready[s][r & 1]));
            // valid columns of the last selected tile (only the last key tile is ragged)
            int last_valid = p.tk;
            if (p.k > 0) {
                const int jl = p.dense ? p.Tk - 1 : __ldg(list + p.k - 1);
                if (jl == p.Tk - 1) last_valid = p.n_last;
            }
            float m = -INFINITY;  // running max of the log2-domain logits (lazy)
            float l = 0.f;        // running sum of 2^(x - m)
            // One step (key tile or landmark chunk j), as a generic lambda so that
            // the selected tiles and the landmark chunks each get a loop of
            // their own (the selected-tile loop holds no landmark code).
            auto step = [&](auto lm_tag, int j) -> bool {
                constexpr bool is_lm = decltype(lm_tag)::value;
                if (!mbar_wait_warp(smem_addr(&b.s_full), ph, wc)) return false;
                tc_fence_after();
                float x[BN];
                {
                    uint32_t raw[BN];
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c) tmem_ld32(tm_s + c * 32, sub32(raw, c * 32));
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c) tmem_wait_ld_dep(sub32(raw, c * 32));
#pragma unroll
                    for (int e = 0; e < BN; ++e) x[e] = __uint_as_float(raw[e]);
                }
                tc_fence_before();
                mbar_arrive(smem_addr(&b.s_free));  // S is in registers: the next Q K^T may overwrite it
                if constexpr (!is_lm) {
                    // selected tile: mask the columns past the tile's length
                    const int valid = (j == p.k - 1) ? last_valid : p.tk;
                    if (valid < BN) {
#pragma unroll
                        for (int e = 0; e < BN; ++e)
                            if (e >= valid) x[e] = -INFINITY;
                    }
                } else {
                    // landmark chunk: x = s * scale + log2(t), or -inf for selected
                    // tiles (from the item's bitmap) and for columns past the last
                    // tile; the ragged last tile's landmark (in the item's last
                    // chunk) then gets log2(n_last) instead
                    const int j0 = (j - p.k) * BN;
                    if (j == p.k) {  // first landmark step: every thread's bits are in
                        if (!mbar_wait_warp(smem_addr(&sm.bm_ready[s][r & 1]), (r >> 1) & 1, wc)) return false;
                    }
                    uint32_t bits[BN / 32];
#pragma unroll
                    for (int w = 0; w < BN / 32; ++w) {
                        const int jw = j0 + w * 32;
                        bits[w] = jw < p.Tk ? bm[jw >> 5] : 0u;
                        const int keep = p.Tk - jw;  // columns >= keep are beyond the last tile
                        if (keep < 32) bits[w] |= keep <= 0 ? 0xFFFFFFFFu : (0xFFFFFFFFu << keep);
                    }
                    const float lt = p.log2_tk;
#pragma unroll
                    for (int w = 0; w < BN / 32; ++w) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float b0 = ((bits[w] >> e) & 1u) ? -INFINITY : lt;
                            const float b1 = ((bits[w] >> (e + 1)) & 1u) ? -INFINITY : lt;
                            float v0, v1;
                            f2_unpack(f2_fma(f2_pack(x[w * 32 + e], x[w * 32 + e + 1]), c2, f2_pack(b0, b1)), v0, v1);
                            x[w * 32 + e] = v0;
                            x[w * 32 + e + 1] = v1;
                        }
                    }
                    if (j == n - 1 && p.n_last != p.tk) {  // once per item
                        const int lastc = p.Tk - 1 - j0;
                        const float dl = p.log2_last - p.log2_tk;
#pragma unroll
                        for (int e = 0; e < BN; ++e) x[e] += e == lastc ? dl : 0.f;
                    }
                }
                // ---- row max: a tree of 3-input max (selected tiles: of the
                // raw scores, scaled afterwards, as scale > 0)
                float mx;
                {
                    float gq[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float t = fmax3(x[16 * q], x[16 * q + 1], x[16 * q + 2]);
#pragma unroll
                        for (int e = 3; e < 15; e += 2) t = fmax3(t, x[16 * q + e], x[16 * q + e + 1]);
                        gq[q] = fmaxf(t, x[16 * q + 15]);
                    }
                    mx = fmax3(fmax3(gq[0], gq[1], gq[2]), fmax3(gq[3], gq[4], gq[5]), fmaxf(gq[6], gq[7]));
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
                const uint64_t nm2 = f2_pack(nm, nm);
                const uint64_t cm2 = is_lm ? f2_pack(1.f, 1.f) : c2;  // landmark logits are already scaled
                // ---- p = 2^(x * scale - m): packed fp32x2 scaling, 2^x on MUFU, two
                // partial row sums, P as bf16 pairs kept in registers until the
                // previous P V is done
                uint64_t acc0 = 0ull, acc1 = 0ull;
                uint32_t pk[BN / 2];
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) {
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const uint64_t xs = f2_fma(f2_pack(x[c * 32 + 2 * q], x[c * 32 + 2 * q + 1]), cm2, nm2);
                        float a0, a1;
                        f2_unpack(xs, a0, a1);
                        const uint64_t pv = f2_pack(ex2(a0), ex2(a1));
                        if (q & 1) acc1 = f2_add(acc1, pv); else acc0 = f2_add(acc0, pv);
                        float p0, p1;
                        f2_unpack(pv, p0, p1);
                        pk[c * 16 + q] = pack_bf16x2(p0, p1);
                    }
                }
                {
                    float s0, s1;
                    f2_unpack(f2_add(acc0, acc1), s0, s1);
                    l += s0 + s1;
                }
                // P is free once P V of the previous step is done; O then holds
                // every earlier step and can be rescaled (the exponentials above
                // overlap that P V)
                if (!mbar_wait_warp(smem_addr(&b.p_free), ph ^ 1u, wc)) return false;
                tc_fence_after();
                // the rescale is decided per row, but tcgen05.ld / st are warp-collective:
                // the whole warp takes the branch and rows without a rescale multiply by 1
                if (__any_sync(0xffffffffu, rescale && j > 0)) {
                    const float a = (rescale && j > 0) ? alpha : 1.f;
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t ro[32];
                        tmem_ld32(tm_o + c * 32, ro);
                        tmem_wait_ld_dep(ro);
#pragma unroll
                        for (int e = 0; e < 32; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * a);
                        tmem_st32(tm_o + c * 32, ro);
                        tmem_wait_st();
                    }
                }
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) tmem_st16(tm_p + c * 16, pk + c * 16);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_addr(&b.p_full));
                return true;
            };
            for (int j = 0; j < p.k && ok; ++j, ph ^= 1u) ok = step(std::false_type{}, j);
            if constexpr (LM) {
                for (int j = p.k; j < n && ok; ++j, ph ^= 1u) ok = step(std::true_type{}, j);
            }
            if (!ok) break;
            // ------------------------------------------------ epilogue ----
            // P V of the item's last step (parity ph ^ 1) has completed, so every
            // thread of the slot is past its landmark steps: clear this item's bits
            if (!mbar_wait_warp(smem_addr(&b.p_free), ph ^ 1u, wc)) { ok = false; break; }
            tc_fence_after();
            if (list && p.lm_chunks) {
                for (int q = row; q < p.k; q += BM) {
                    const int t = __ldg(list + q);
                    const int tc = t < 0 ? 0 : (t >= p.Tk ? p.Tk - 1 : t);
                    atomicAnd(&bm[tc >> 5], ~(1u << (tc & 31)));
                }
            }
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
            mbar_arrive(smem_addr(&b.o_free));
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
                             unsigned* wave, cudaStream_t st) {
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
    p.wave = wave;
    p.status = dev.status;
    p.timeout_ns = wait_timeout_ns();
    // The setmaxnreg split only adds up for a kernel compiled to exactly
    // LAUNCH_REGS registers per thread; refuse to launch anything else.
    static int regs_ok = -1;
    static std::mutex regs_mu;
    {
        std::lock_guard<std::mutex> lock(regs_mu);
        if (regs_ok < 0) {
            cudaFuncAttributes fa, fb;
            if (cudaFuncGetAttributes(&fa, sparse_attn_kernel<true>) != cudaSuccess) return ZB_ERR_CUDA;
            if (cudaFuncGetAttributes(&fb, sparse_attn_kernel<false>) != cudaSuccess) return ZB_ERR_CUDA;
            regs_ok = (fa.numRegs == LAUNCH_REGS && fb.numRegs == LAUNCH_REGS) ? 1 : 0;
        }
        if (!regs_ok) return ZB_ERR_UNSUPPORTED;
    }
    const void* kern = lm_chunks ? reinterpret_cast<const void*>(sparse_attn_kernel<true>)
                                 : reinterpret_cast<const void*>(sparse_attn_kernel<false>);
    const size_t smem = attn_smem_bytes();
    cudaError_t ce = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (ce != cudaSuccess) return ZB_ERR_CUDA;
    const long long grid = p.n_items < dev.sm_count ? p.n_items : dev.sm_count;
    if (!wave) {
        if (lm_chunks)
            sparse_attn_kernel<true><<<static_cast<unsigned>(grid), NUM_THREADS, smem, st>>>(mq, mk, mv, mkb, mvb, p);
        else
            sparse_attn_kernel<false><<<static_cast<unsigned>(grid), NUM_THREADS, smem, st>>>(mq, mk, mv, mkb, mvb, p);
        return cudaGetLastError() == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
    }
    // The wave barriers need every CTA resident at once: zero the counters in
    // stream order, then a cooperative launch (which guarantees co-residency).
    if (cudaMemsetAsync(wave, 0, sizeof(unsigned), st) != cudaSuccess) return ZB_ERR_CUDA;
    void* args[] = {&mq, &mk, &mv, &mkb, &mvb, &p};
    ce = cudaLaunchCooperativeKernel(kern, dim3(static_cast<unsigned>(grid)), dim3(NUM_THREADS), args, smem, st);
    return ce == cudaSuccess ? ZB_OK : ZB_ERR_CUDA;
}

}  // namespace zb

using namespace zb;

extern "C" size_t zb_tile_sparse_attn_workspace_bytes(void) { return 256; }

extern "C" zb_status zb_tile_sparse_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                         const uint16_t* Kbar_bf16, const uint16_t* Vbar_bf16,
                                         const int32_t* idx, int32_t k, int32_t use_landmarks,
                                         float scale, zb_shape s, uint16_t* O, float* lse,
                                         void* ws, size_t ws_bytes, void* stream) {
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
        !aligned16(lse) || !aligned16(ws) || (lm && (!aligned16(Kbar_bf16) || !aligned16(Vbar_bf16))))
        return ZB_ERR_ALIGN;
    if (ws && ws_bytes < zb_tile_sparse_attn_workspace_bytes()) return ZB_ERR_WORKSPACE;
    return launch_attn(Q, K, V, Kbar_bf16, Vbar_bf16, idx, s.heads, s.n_tokens, s.n_tokens, s.tile,
                       s.tile, k, 0, use_landmarks ? 1 : 0, scale, O, 0, lse, static_cast<unsigned*>(ws),
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
                       scale, O, out_fp32 ? 1 : 0, lse, nullptr, static_cast<cudaStream_t>(stream));
}
