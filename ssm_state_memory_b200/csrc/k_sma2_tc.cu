// State-memory attention forward on a pair of SMs (tcgen05 cta_group::2), sm_100a.
//
// The same computation as k_sma_fwd_tc (DART §3 eq 8-10, §4 Algorithm 1, App. C eq 28-31 online
// softmax), for chunks of a multiple of 256 tokens, run by clusters of two CTAs on the two SMs of a TPC:
//
//   work item = (chunk i, batch row, 256-token tile pair of the chunk, group of 4 (or 2) heads). CTA rank r
//               of the pair owns the tile 2 * pair + r: its 128 rows of Q and C stay in its shared memory.
//   product   = per head pair (h, h+1) and chunk step j < i, the leader (rank 0) issues M = 256 products
//               Q [dH_h[j] | dH_h+1[j]] and C [dH_h[j] | dH_h+1[j]] (N = 128, K = 16 each): A is each
//               CTA's own Q or C tile, and the B columns are split, dH_h[j] in the leader's shared memory
//               and dH_h+1[j] in the peer's. Each CTA's tensor memory receives its own 128 rows of both
//               heads, double-buffered as in the one-SM kernel.
//   why       = a one-SM M = 128, N = 128 product reads 8 KiB of operands from shared memory per K = 16
//               step, and with the chunk-memory stream arriving by TMA at the same time the kernel was
//               bound by shared-memory bandwidth at about 78% of the tensor pipe's rate in steady state.
//               Per SM the pair reads A (4 KiB) and half of B (2 KiB) per step, and each CTA loads only
//               one head's chunk memory per step (16 KiB instead of 32).
//   loads     = each CTA's producer loads its own tiles into its own shared memory and counts them on its
//               own barrier (no TMA multicast). A relay thread in the peer forwards the completion of each
//               of its loads to the leader, which issues a step once both halves are in. So every CTA
//               waits for exactly the copies it started before it exits.
//   softmax   = warps 4-11 of each CTA, one token row per thread, exactly as in the one-SM kernel; they
//               free a tensor-memory buffer by arriving on the leader's barrier (16 arrivals).
//
// Tokens of chunk 0 (no history) get R = 0 and lse = -inf (eq 10 text).
#include <cuda.h>
#include <math.h>

#include <algorithm>

#include "dart_internal.cuh"
#include "sm100_ptx.cuh"

namespace dart {
namespace {

using namespace sm100;

constexpr int kThreads = 384;     // 12 warps = 3 warpgroups
constexpr int kRegsLaunch = 168;  // registers per thread the kernel must be launched with
constexpr int kRegsLow = 80;      // warpgroup 0 (producer, MMA issuer or relay, two idle warps)
constexpr int kRegsHigh = 208;    // warpgroups 1-2 (softmax)
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kRegsLaunch, "register split exceeds the pool");
constexpr int kStages = 4;        // dH ring depth (one stage = this CTA's head of a pair: one box)
constexpr int kTileRows = 128;
constexpr int kN = 128;
constexpr int kP = 64;
constexpr uint32_t kBox = 128 * 128;            // one 128-row x 64-col bf16 TMA box = 16 KiB
constexpr uint32_t kQOff = 0;                   // Q tile: [k-half 0..1] boxes
constexpr uint32_t kCOff = 2 * kBox;            // C tile: same
constexpr uint32_t kHOff = 4 * kBox;            // dH stages: one box each
constexpr uint32_t kStgOff = kHOff + kStages * kBox;  // per softmax warp two 32 x 128-byte tiles
constexpr uint32_t kBarOff = kStgOff + 8 * 8192;
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O and d may grow by at most 2^8 before rescaling

// L*: this CTA's own loads have landed. P*: (leader only) the peer's loads have landed, forwarded by the
// peer's relay thread. *_EMPTY and TMEM_FULL: arrived by the leader's tensor-core commits, in both CTAs.
// TMEM_EMPTY (leader only): the 16 softmax warps of the pair have read a buffer.
enum {
    BAR_LQC_FULL = 0, BAR_PQC_FULL, BAR_QC_EMPTY, BAR_MMA_DONE, BAR_LSTAGE_FULL, BAR_PSTAGE_FULL = BAR_LSTAGE_FULL + kStages,
    BAR_STAGE_EMPTY = BAR_PSTAGE_FULL + kStages, BAR_TMEM_FULL = BAR_STAGE_EMPTY + kStages,
    BAR_TMEM_EMPTY = BAR_TMEM_FULL + 2, BAR_E_FULL = BAR_TMEM_EMPTY + 2, BAR_COUNT = BAR_E_FULL + 8
};
static_assert(BAR_COUNT * 8 + 8 <= 256, "barrier block overflows its 256 bytes");

struct Sma2Params {
    Shape s;
    int hpi;         // heads per work item (2 or 4, dividing H / G)
    int npairs;      // 256-token tile pairs per chunk (S / 256)
    int ngh;         // head groups per batch row = H / hpi
    int64_t n_items;
    float *out;      // R; with combine, out (holding Y on entry), to which g R is added
    float *lse;
    const float *g;
    int64_t g_sb, g_st, g_sh;
    int combine;
    int hpe_log2;    // log2 of the heads per E group (0: E per head)
    int *err;        // device error word (first member of the device control block)
};

struct Item {
    int64_t i, b, pair, hg;
};

// Items sorted longest first: (chunk i descending, batch row, tile pair, head group).
__device__ __forceinline__ Item decode_item(const Sma2Params &p, int64_t k) {
    const uint32_t ngh = (uint32_t)p.ngh, per_b = (uint32_t)p.npairs * ngh, per_i = (uint32_t)p.s.Bt * per_b;
    const uint32_t k32 = (uint32_t)k;
    Item it;
    const uint32_t q = k32 / per_i;
    it.i = p.s.M - 1 - (int64_t)q;
    uint32_t r = k32 - q * per_i;
    const uint32_t b = r / per_b;
    r -= b * per_b;
    const uint32_t pr = r / ngh;
    it.b = b;
    it.pair = pr;
    it.hg = r - pr * ngh;
    return it;
}

// first token of tile `tile` (0 or 1) of the item's pair
__device__ __forceinline__ int64_t tile_t0(const Sma2Params &p, const Item &it, int tile) {
    return it.i * p.s.S + (2 * it.pair + tile) * kTileRows;
}

__device__ __forceinline__ int tile_rows(const Sma2Params &p, const Item &it, int tile) {
    const int64_t end = min(p.s.L, (it.i + 1) * p.s.S);
    return (int)max((int64_t)0, min((int64_t)kTileRows, end - tile_t0(p, it, tile)));
}

// The tile whose rows CTA `rank` loads: its own, or the first one when its own lies wholly past the end of
// the batch row (the CTA then computes on those rows and stores nothing), so no load is wholly out of bounds.
__device__ __forceinline__ int load_tile(const Sma2Params &p, const Item &it, int rank) {
    return tile_rows(p, it, rank) > 0 ? rank : 0;
}

// An item the pair computes: it has history and its first tile has rows (the second may be empty past a
// ragged end; its CTA then runs on zero-filled or unused rows and stores nothing).
__device__ __forceinline__ bool item_live(const Sma2Params &p, const Item &it) {
    return it.i > 0 && tile_rows(p, it, 0) > 0;
}

// Item order per cluster, as sched_next per CTA: alternating direction over the G clusters each round.
__device__ __forceinline__ int64_t sched_next_pair(int64_t k) {
    const uint32_t g = gridDim.x >> 1, k32 = (uint32_t)k;
    const uint32_t m = k32 / g, r = k32 - m * g;
    return (int64_t)(m + 2) * g - 1 - r;
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
    k_sma_fwd_pair_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC,
                      const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmE,
                      const __grid_constant__ CUtensorMap tmR, const Sma2Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kBarOff);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kBarOff + BAR_COUNT * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kBarOff + BAR_COUNT * 8 + 4);
    auto bar = [&](int k) { return smem_u32(&bars[k]); };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int64_t cid = blockIdx.x >> 1;
    if (threadIdx.x == 0) {
        mbar_init(bar(BAR_LQC_FULL), 1);
        mbar_init(bar(BAR_PQC_FULL), 1);
        mbar_init(bar(BAR_QC_EMPTY), 1);
        mbar_init(bar(BAR_MMA_DONE), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(BAR_LSTAGE_FULL + s), 1);
            mbar_init(bar(BAR_PSTAGE_FULL + s), 1);
            mbar_init(bar(BAR_STAGE_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(BAR_TMEM_FULL + b), 1);
            mbar_init(bar(BAR_TMEM_EMPTY + b), 16);  // one arrival per softmax warp of the pair
        }
        for (int w = 0; w < 8; ++w) mbar_init(bar(BAR_E_FULL + w), 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmH);
        tma_prefetch_desc(&tmR);
        tma_prefetch_desc(&tmE);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers are initialised and their tensor memory allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int *err = p.err;
    const Shape &s = p.s;

    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        setmaxnreg_dec<kRegsLow>();
        if (lane == 0) {
            uint32_t qc_uses = 0;
            int st = 0;            // ring slot of the next load
            uint32_t ph = 0;       // parity of the ring's current pass
            int last_ph[kStages];  // parity of the last load into each slot (-1: none)
            for (int q = 0; q < kStages; ++q) last_ph[q] = -1;
            bool qc_loaded = false;
            for (int64_t k = cid; k < p.n_items; k = sched_next_pair(k)) {
                const Item it = decode_item(p, k);
                if (!item_live(p, it)) continue;
                const int64_t h0 = it.hg * p.hpi;
                const int64_t grp = h0 / (s.H / s.G);
                if (!mbar_wait(bar(BAR_QC_EMPTY), (qc_uses & 1) ^ 1, abort_flag, err, 211)) goto producer_end;
                mbar_arrive_expect_tx(bar(BAR_LQC_FULL), 4 * kBox);
                {
                    const int32_t y = (int32_t)(it.b * s.L + tile_t0(p, it, load_tile(p, it, (int)rank)));
                    for (int kh = 0; kh < 2; ++kh) {
                        const int32_t x = (int32_t)(grp * kN + kh * 64);
                        tma_load_2d(sbase + kQOff + kh * kBox, &tmQ, x, y, bar(BAR_LQC_FULL));
                        tma_load_2d(sbase + kCOff + kh * kBox, &tmC, x, y, bar(BAR_LQC_FULL));
                    }
                }
                ++qc_uses;
                qc_loaded = true;
                for (int hp = 0; hp < p.hpi; hp += 2) {
                    const int64_t h = h0 + hp + rank;  // this CTA's head of the pair
                    for (int64_t j = 0; j < it.i; ++j) {
                        if (!mbar_wait(bar(BAR_STAGE_EMPTY + st), ph ^ 1, abort_flag, err, 212)) goto producer_end;
                        mbar_arrive_expect_tx(bar(BAR_LSTAGE_FULL + st), kBox);
                        tma_load_2d(sbase + kHOff + st * kBox, &tmH, 0, (int32_t)(((it.b * s.H + h) * s.M + j) * kN),
                                    bar(BAR_LSTAGE_FULL + st));
                        last_ph[st] = (int)ph;
                        if (++st == kStages) {
                            st = 0;
                            ph ^= 1;
                        }
                    }
                }
            }
        producer_end:
            // never leave a copy in flight into shared memory that is about to be released
            for (int q = 0; q < kStages; ++q)
                if (last_ph[q] >= 0) mbar_drain(bar(BAR_LSTAGE_FULL + q), (uint32_t)last_ph[q]);
            if (qc_loaded) mbar_drain(bar(BAR_LQC_FULL), (qc_uses - 1) & 1);
        }
    } else if (warp == 1) {
        setmaxnreg_dec<kRegsLow>();
        if (lane == 0 && rank == 1) {
            // ------------------------- relay (peer CTA) --------------------------
            // Forwards the completion of each of this CTA's loads to the leader's P* barrier, in the order the
            // leader consumes them.
            const uint32_t pqc = mapa_shared(bar(BAR_PQC_FULL), 0);
            uint32_t qc_uses = 0;
            int st = 0;
            uint32_t ph = 0;
            for (int64_t k = cid; k < p.n_items; k = sched_next_pair(k)) {
                const Item it = decode_item(p, k);
                if (!item_live(p, it)) continue;
                if (!mbar_wait(bar(BAR_LQC_FULL), qc_uses & 1, abort_flag, err, 221)) goto relay_end;
                ++qc_uses;
                mbar_arrive_cluster(pqc);
                for (int hp = 0; hp < p.hpi; hp += 2) {
                    for (int64_t j = 0; j < it.i; ++j) {
                        if (!mbar_wait(bar(BAR_LSTAGE_FULL + st), ph, abort_flag, err, 222)) goto relay_end;
                        mbar_arrive_cluster(mapa_shared(bar(BAR_PSTAGE_FULL + st), 0));
                        if (++st == kStages) {
                            st = 0;
                            ph ^= 1;
                        }
                    }
                }
            }
        relay_end:;
        } else if (lane == 0) {
            // -------------------------------- MMA (leader) --------------------------------
            // M = 256 (the pair's two tiles), N = 128 = the pair's two heads (one per CTA's B half), A K-major,
            // B MN-major (one 64-column box in each CTA)
            constexpr uint32_t idesc = idesc_bf16_f32(2 * kTileRows, 2 * kP, false, true);
            const uint64_t qdesc0 = smem_desc_sw128(sbase + kQOff, 16, 1024);
            const uint64_t cdesc0 = smem_desc_sw128(sbase + kCOff, 16, 1024);
            uint32_t qc_uses = 0, tb = 0;
            int st = 0;
            uint32_t ph = 0;
            bool issued = false;
            for (int64_t k = cid; k < p.n_items; k = sched_next_pair(k)) {
                const Item it = decode_item(p, k);
                if (!item_live(p, it)) continue;
                if (!mbar_wait(bar(BAR_LQC_FULL), qc_uses & 1, abort_flag, err, 231)) goto mma_end;
                if (!mbar_wait_cluster(bar(BAR_PQC_FULL), qc_uses & 1, abort_flag, err, 232)) goto mma_end;
                ++qc_uses;
                tc_fence_after();
                for (int hp = 0; hp < p.hpi; hp += 2) {
                    for (int64_t j = 0; j < it.i; ++j) {
                        if (!mbar_wait(bar(BAR_LSTAGE_FULL + st), ph, abort_flag, err, 233)) goto mma_end;
                        if (!mbar_wait_cluster(bar(BAR_PSTAGE_FULL + st), ph, abort_flag, err, 234)) goto mma_end;
                        const int buf = tb & 1;
                        if (!mbar_wait_cluster(bar(BAR_TMEM_EMPTY + buf), ((tb >> 1) & 1) ^ 1, abort_flag, err, 235))
                            goto mma_end;
                        tc_fence_after();
                        const uint64_t bdesc0 = smem_desc_sw128(sbase + kHOff + st * kBox, kBox, 1024);
                        const uint32_t dq = tmem + buf * 256;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t aoff = (uint64_t)((((kk >> 2) * kBox) + (kk & 3) * 32) >> 4);
                            const uint64_t bdesc = bdesc0 + (uint64_t)((kk * 2048) >> 4);
                            mma_bf16_pair(dq, qdesc0 + aoff, bdesc, idesc, kk > 0);
                            mma_bf16_pair(dq + 128, cdesc0 + aoff, bdesc, idesc, kk > 0);
                        }
                        mma_commit_pair(bar(BAR_STAGE_EMPTY + st), 3);
                        mma_commit_pair(bar(BAR_TMEM_FULL + buf), 3);
                        issued = true;
                        if (++st == kStages) {
                            st = 0;
                            ph ^= 1;
                        }
                        ++tb;
                    }
                }
                mma_commit_pair(bar(BAR_QC_EMPTY), 3);
            }
        mma_end:
            if (issued) {  // every issued product has finished before tensor memory is released
                mma_commit_pair(bar(BAR_MMA_DONE), 1);
                mbar_drain(bar(BAR_MMA_DONE), 0);
            }
        }
    } else if (warp < 4) {
        setmaxnreg_dec<kRegsLow>();  // no role, registers only
    } else {
        // ------------------------------ softmax -------------------------------
        setmaxnreg_inc<kRegsHigh>();
        const int e = (warp - 4) >> 2;  // warpgroup = head of the pair
        const int quarter = warp & 3;   // tensor-memory lane quarter this warp may access
        const int row = quarter * 32 + lane;
        const float escale = kLog2e * rsqrtf((float)kN);
        const uint32_t tmem_empty[2] = {mapa_shared(bar(BAR_TMEM_EMPTY), 0), mapa_shared(bar(BAR_TMEM_EMPTY + 1), 0)};
        uint32_t tb = 0;
        // This warp's two 4 KiB tiles: tile 0 carries, in turn, the E rows of the next pair (TMA load, issued
        // one chunk into the current pair) and the first column half of the current pair's R rows (TMA store
        // at its end); tile 1 the second half.
        uint8_t *stg = sm + kStgOff + (warp - 4) * 8192;
        const uint32_t ebar = bar(BAR_E_FULL + (warp - 4));
        uint32_t ev[kP / 2];              // E_t of the current pair (bf16 pairs)
        int64_t ev_k = -1, pend_k = -1;   // pair whose E is in ev / in flight into the tile
        int ev_hp = 0, pend_hp = 0;
        uint32_t e_uses = 0;
        // E rows of pair (k2, hp2) into the tile, once its previous R stores have read it
        auto issue_e = [&](int64_t k2, int hp2) {
            if (k2 >= p.n_items) return;
            const Item it2 = decode_item(p, k2);
            if (!item_live(p, it2)) return;
            __syncwarp();  // every lane is done with the tile's previous contents
            if (lane == 0) {
                bulk_wait_group_read<0>();
                fence_async_smem();
                mbar_arrive_expect_tx(ebar, 4096);
                tma_load_3d(smem_u32(stg), &tmE, (int32_t)((((int)it2.hg * p.hpi + hp2 + e) >> p.hpe_log2) * kP),
                            (int32_t)(tile_t0(p, it2, load_tile(p, it2, (int)rank)) + quarter * 32), (int32_t)it2.b,
                            ebar);
            }
            pend_k = k2;
            pend_hp = hp2;
        };
        // the pending E rows into ev; false when the wait gave up
        auto take_e = [&]() -> bool {
            if (!mbar_wait(ebar, e_uses & 1, abort_flag, err, 241)) return false;
            ++e_uses;
            const uint8_t *srow = stg + lane * 128;
#pragma unroll
            for (int q = 0; q < kP / 8; ++q) {
                const uint4 v = *reinterpret_cast<const uint4 *>(srow + ((q ^ (lane & 7)) << 4));
                ev[4 * q] = v.x;
                ev[4 * q + 1] = v.y;
                ev[4 * q + 2] = v.z;
                ev[4 * q + 3] = v.w;
            }
            __syncwarp();
            ev_k = pend_k;
            ev_hp = pend_hp;
            pend_k = -1;
            return true;
        };
        for (int64_t k = cid; k < p.n_items; k = sched_next_pair(k)) {
            const Item it = decode_item(p, k);
            const int rows = tile_rows(p, it, (int)rank);
            const int64_t t0 = tile_t0(p, it, (int)rank);
            const int64_t t = t0 + row;
            const bool valid = row < rows;
            const bool live = item_live(p, it);
            if (!live && rows == 0) continue;  // nothing of this tile exists
            for (int hp = 0; hp < p.hpi; hp += 2) {
                const int64_t h = it.hg * p.hpi + hp + e;
                if (!live) {  // chunk 0: no historical chunk for any row of the tile
                    if (valid) {
                        if (!p.combine) {
                            float4 *o4 = reinterpret_cast<float4 *>(p.out + ((it.b * s.L + t) * s.H + h) * kP);
#pragma unroll
                            for (int q = 0; q < kP / 4; ++q) o4[q] = make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                        if (p.lse) p.lse[(it.b * s.H + h) * s.L + t] = -INFINITY;
                    }
                    continue;
                }
                // E_t (bf16 pairs) stays in registers for the whole chunk loop
                if (ev_k != k || ev_hp != hp) {  // not fetched ahead (first pair, or after items without history)
                    if (pend_k >= 0 && !take_e()) goto softmax_end;
                    issue_e(k, hp);
                    if (!take_e()) goto softmax_end;
                }
                // fused layer: this row's gate, fetched before the chunk loop
                const float gate = (p.combine && valid) ? __ldg(p.g + it.b * p.g_sb + t * p.g_st + h * p.g_sh) : 0.f;
                int64_t nk = k;  // the next pair
                int nhp = hp + 2;
                if (nhp >= p.hpi) {
                    nhp = 0;
                    nk = sched_next_pair(k);
                }
                float O[kP];
#pragma unroll
                for (int q = 0; q < kP; ++q) O[q] = 0.f;
                float m = -INFINITY, d = 0.f;
                for (int64_t j = 0; j < it.i; ++j) {
                    const int buf = tb & 1;
                    if (!mbar_wait(bar(BAR_TMEM_FULL + buf), (tb >> 1) & 1, abort_flag, err, 242)) goto softmax_end;
                    tc_fence_after();
                    const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + buf * 256 + e * kP;
                    // logit: (Q_t dH[j]) . E_t, read in two 32-column halves, four partial sums
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float u[32];
                        tmem_ld_32x32b_x32_after(ta + half * 32, u, acc[0]);
                        tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const uint32_t w = ev[16 * half + q];
                            acc[q & 3] = fmaf(u[2 * q], __uint_as_float(w << 16), acc[q & 3]);
                            acc[q & 3] = fmaf(u[2 * q + 1], __uint_as_float(w & 0xffff0000u), acc[q & 3]);
                        }
                    }
                    const float l2 = ((acc[0] + acc[1]) + (acc[2] + acc[3])) * escale;  // l_{t,j}, log2 units
                    if (l2 > m + kRescaleThreshold) {  // lazy rescale: only when the running max grows a lot
                        const float f = exp2f(m - l2);
                        d *= f;
#pragma unroll
                        for (int q = 0; q < kP; ++q) O[q] *= f;
                        m = l2;
                    }
                    __syncwarp();  // reconverge before the warp-collective tensor-memory loads
                    const float pw = exp2f(l2 - m);
                    d += pw;
                    // value C_t dH[j], accumulated with weight pw
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float v[32];
                        tmem_ld_32x32b_x32_after(ta + 128 + half * 32, v, pw + O[32 * half]);
                        tmem_ld_wait();
                        if (half == 1) {  // both halves read: hand the buffer back to the leader's MMA early
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive_cluster(tmem_empty[buf]);
                        }
#pragma unroll
                        for (int q = 0; q < 32; ++q) O[32 * half + q] = fmaf(pw, v[q], O[32 * half + q]);
                    }
                    ++tb;
                    if (j == 0) issue_e(nk, nhp);  // a chunk in, the previous pair's R stores are done
                }
                // the next pair's E rows out of the tile before R goes through it
                if (pend_k >= 0 && !take_e()) goto softmax_end;
                {
                    // R = O / d through this warp's staging tiles, 32 rows x 32 columns each, by TMA store; in
                    // the fused layer (combine) g R instead, added into out (which holds Y) by a TMA
                    // reduction, eq (11). Either way rows past the end of the batch row are clipped.
                    const float inv = 1.f / d;
                    const float sc = p.combine ? gate * inv : inv;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        if (half == 0 && lane == 0) bulk_wait_group_read<0>();
                        __syncwarp();
                        uint8_t *srow = stg + half * 4096 + lane * 128;
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            *reinterpret_cast<float4 *>(srow + ((q ^ (lane & 7)) << 4)) =
                                make_float4(O[32 * half + 4 * q] * sc, O[32 * half + 4 * q + 1] * sc,
                                            O[32 * half + 4 * q + 2] * sc, O[32 * half + 4 * q + 3] * sc);
                        fence_async_smem();
                        __syncwarp();
                        if (lane == 0 && rows > 0) {  // a tile wholly past the end stores nothing
                            const int32_t tx = (int32_t)(h * kP + half * 32);
                            const int32_t ty = (int32_t)(t0 + quarter * 32);
                            if (p.combine)
                                tma_reduce_add_3d(&tmR, smem_u32(stg + half * 4096), tx, ty, (int32_t)it.b);
                            else
                                tma_store_3d(&tmR, smem_u32(stg + half * 4096), tx, ty, (int32_t)it.b);
                            bulk_commit_group();
                        }
                    }
                }
                if (valid && p.lse) p.lse[(it.b * s.H + h) * s.L + t] = (m + log2f(d)) * kLn2;
            }
        }
    softmax_end:
        if (pend_k >= 0) mbar_drain(ebar, e_uses & 1);  // an E load still in flight into the tile
        if (lane == 0) bulk_wait_group<0>();            // every R store has landed before the CTA exits
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the leader's products into both CTAs' tensor memory, and every arrival, are done
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace

// S a multiple of 256 (a chunk holds whole tile pairs), H / G even, the plain score branch.
bool pair_tc_shape_ok(const Shape &s, bool bf16) {
    if (!bf16 || s.N != kN || s.P != kP || s.S % (2 * kTileRows) != 0) return false;
    if ((s.H / s.G) % 2 != 0) return false;
    if (s.M * (s.S / (2 * kTileRows)) * s.Bt * (s.H / 2) >= (int64_t(1) << 31)) return false;  // 32-bit decode
    if (s.Bt * s.L >= (int64_t(1) << 31) || s.Bt * s.H * s.M * s.N >= (int64_t(1) << 31)) return false;
    return true;
}

cudaError_t launch_sma_fwd_pair_tc(const Shape &s, const LayerPtrs &lp, cudaStream_t st) {
    Sma2Params p{};
    p.s = s;
    const int64_t hpg = s.H / s.G;
    p.hpi = hpg % 4 == 0 ? 4 : 2;
    p.ngh = (int)(s.H / p.hpi);
    p.npairs = (int)(s.S / (2 * kTileRows));
    p.n_items = s.M * p.npairs * s.Bt * p.ngh;
    p.combine = lp.combine ? 1 : 0;
    p.out = static_cast<float *>(lp.combine ? lp.Y : lp.R);
    p.lse = lp.lse;
    p.g = lp.g;
    p.g_sb = lp.g_sb;
    p.g_st = lp.g_st;
    p.g_sh = lp.g_sh;
    p.err = device_error_word();
    const int64_t hpe = heads_per_e(s, lp.e_groups);  // a power of two on this path
    while ((int64_t(1) << p.hpe_log2) < hpe) ++p.hpe_log2;
    const uint64_t EGP = (uint64_t)(s.H / hpe * s.P);
    CUtensorMap mq, mc, mh, me, mr;
    if (!make_tma_map_bf16(&mq, lp.Q, (uint64_t)(s.G * s.N), (uint64_t)(s.Bt * s.L), (uint64_t)(s.G * s.N * 2), 64,
                           128) ||
        !make_tma_map_bf16(&mc, lp.C, (uint64_t)(s.G * s.N), (uint64_t)(s.Bt * s.L), (uint64_t)(s.G * s.N * 2), 64,
                           128) ||
        !make_tma_map_bf16(&mh, lp.dH, (uint64_t)s.P, (uint64_t)(s.Bt * s.H * s.M * s.N), (uint64_t)(s.P * 2), 64,
                           128) ||
        !make_tma_map_f32_3d(&mr, p.out, (uint64_t)(s.H * s.P), (uint64_t)s.L, (uint64_t)s.Bt, (uint64_t)(s.H * s.P * 4),
                             (uint64_t)(s.L * s.H * s.P * 4), 32, 32) ||
        !make_tma_map_bf16_3d(&me, lp.E, EGP, (uint64_t)s.L, (uint64_t)s.Bt, EGP * 2, (uint64_t)s.L * EGP * 2, 64, 32))
        return cudaErrorInvalidValue;
    static int max_clusters = 0;
    if (!max_clusters) {
        // the register split of the warpgroups assumes this launch size (see k_sma_fwd_tc)
        cudaFuncAttributes fa{};
        cudaError_t ea = cudaFuncGetAttributes(&fa, k_sma_fwd_pair_tc);
        if (ea != cudaSuccess || fa.numRegs != kRegsLaunch) {
            set_last_error("sma_fwd_pair_tc built with an unexpected register count", cudaErrorInvalidConfiguration);
            return ea != cudaSuccess ? ea : cudaErrorInvalidConfiguration;
        }
        cudaError_t e = cudaFuncSetAttribute(k_sma_fwd_pair_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemBytes);
        if (e != cudaSuccess) {
            set_last_error("cudaFuncSetAttribute(sma_fwd_pair_tc)", e);
            return e;
        }
        cudaLaunchConfig_t qc{};
        cudaLaunchAttribute qa[1];
        qa[0].id = cudaLaunchAttributeClusterDimension;
        qa[0].val.clusterDim.x = 2;
        qa[0].val.clusterDim.y = 1;
        qa[0].val.clusterDim.z = 1;
        qc.gridDim = dim3((unsigned)(2 * (device_sm_count() / 2)), 1, 1);
        qc.blockDim = dim3(kThreads, 1, 1);
        qc.dynamicSmemBytes = kSmemBytes;
        qc.attrs = qa;
        qc.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, k_sma_fwd_pair_tc, &qc);
        if (e != cudaSuccess || n <= 0) {
            set_last_error("cudaOccupancyMaxActiveClusters(sma_fwd_pair_tc)", e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
            return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
        }
        max_clusters = n;
    }
    const int64_t clusters = std::min<int64_t>(p.n_items, max_clusters);
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    launch_begin(KK_SMA_FWD_TC, st);
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_sma_fwd_pair_tc, mq, mc, mh, me, mr, p);
    if (e != cudaSuccess) {
        set_last_error("cudaLaunchKernelEx(sma_fwd_pair_tc)", e);
        (void)cudaGetLastError();
    }
    const cudaError_t e2 = launch_end(KK_SMA_FWD_TC, st);
    return e != cudaSuccess ? e : e2;
}

}  // namespace dart
