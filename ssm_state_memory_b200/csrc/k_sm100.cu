// tcgen05 (5th-generation tensor core) kernels of the DART forward path, sm_100a.
//
// State-memory attention forward (DART paper §3 eq 8-10, §4 Algorithm 1,
// App. C eq 28-31 online softmax), restated for Blackwell:
//
//   work item  = (128-token tile of a batch row, group of 4 heads); Q and C are
//                shared by the heads of a group (G = 1 in the paper's MVA-style
//                projections, Fig. 2), so their tiles are loaded once per item and
//                stay in shared memory while the heads stream by. With S a multiple
//                of 128 a tile lies in one chunk i and takes the chunk steps j < i;
//                with S < 128 (S dividing 128: the paper's S = 16, 32, 64) it spans
//                128 / S chunks, takes the steps below its last row's chunk, and each
//                row skips the steps at or after its own chunk.
//   producer   = warp 0: TMA (cp.async.bulk.tensor, 128-byte swizzle) of the Q/C
//                tiles and, per head pair, of dH[b, h, j] and dH[b, h+1, j] for
//                j < i side by side through a 3-stage ring.
//   MMA        = warp 1, one thread: per (head pair, j), two chains of 8
//                tcgen05.mma M=128 N=128 K=16 — Q_tile [dH_h | dH_h+1] and
//                C_tile [dH_h | dH_h+1] — with fp32 accumulators in tensor memory,
//                double-buffered (2 x 256 columns). Two heads per instruction keep
//                the instruction count per flop low: at N=64 the per-instruction
//                overhead, not the tensor pipe, bounded the kernel.
//   softmax    = warps 4-11, one warpgroup per head of the pair: each thread owns one
//                token row and keeps E_t in registers; it reads Q dH[j] (64 fp32) from
//                tensor memory, dots it with E_t to get the logit l_{t,j} (eq 9), reads
//                the value C_t dH[j] (eq 8), and folds both into its online-softmax state
//                (m, d, O[64]) with lazy rescaling. The epilogue writes R = O / d and
//                lse = m + log d; in the fused layer, where out already holds the SSD
//                output Y, it adds g R into out by a TMA reduction (eq 11).
//   memory     = every global access of the softmax warps except lse goes through TMA:
//                E rows arrive one pair ahead in a per-warp shared-memory tile and R
//                leaves through two such tiles. Per-lane loads and stores of 128-byte
//                rows 4 KiB apart would split each warp instruction into 32 line
//                requests, and those stalled the head-pair boundaries, where the MMA
//                (only two accumulator buffers ahead) waits for the softmax.
//   registers  = warps 2-3 have no role; warpgroup 0 gives up registers (setmaxnreg)
//                so that the softmax warpgroups hold O, E and a value row at once.
//   normalised = the normalised score branch (App. B.1) adds a fourth warpgroup, warps
//                12-15, that rescales the staged key rows between the value and key
//                chains; the block is then 512 threads of 128 registers at launch.
//
// Tokens of chunk 0 (no history) get R = 0 and lse = -inf (eq 10 text).
#include <cuda.h>
#include <math.h>

#include <algorithm>
#include <cstdio>

#include <cuda_fp16.h>

#include "dart_internal.cuh"
#include "sm100_ptx.cuh"

namespace dart {

__device__ sm100::DevCtl g_dart_ctl = {0, 0, sm100::kWaitNs};
__device__ int g_dart_fp16_range = 0;

namespace {

using namespace sm100;

constexpr int kTcThreads = 384;   // 12 warps = 3 warpgroups
constexpr int kRegsLaunch = 168;  // registers per thread the kernel must be launched with
constexpr int kRegsLow = 80;      // warpgroup 0 (producer, MMA issuer, two idle warps)
constexpr int kRegsHigh = 208;   // warpgroups 1-2 (softmax)
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kTcThreads * kRegsLaunch, "register split exceeds the pool");
// normalised branch: a fourth warpgroup (warps 12-15) rescales the keys, one warp on each scheduler
// (measured at the 8192-token workload: 80 / 80 / 176 took 0.82 ms, 48 / 48 / 208 0.86 ms, the 12-warp
// kernel with two scaler warps 1.08 ms)
constexpr int kTcThreadsNorm = 512;
constexpr int kRegsLaunchNorm = 128;
constexpr int kRegsLowNorm = 80;     // warpgroup 0
constexpr int kRegsHighNorm = 176;   // warpgroups 1-2 (softmax)
constexpr int kRegsScaler = 80;      // warpgroup 3
static_assert(128 * (kRegsLowNorm + kRegsScaler) + 256 * kRegsHighNorm <= kTcThreadsNorm * kRegsLaunchNorm,
              "register split of the normalised kernel exceeds the pool");
constexpr int kStages = 3;        // dH ring depth (one stage = a head pair's chunk memories)
constexpr int kTileRows = 128;    // tokens per MMA tile (M)
constexpr int kN = 128;           // state size (K of the MMA)
constexpr int kP = 64;            // head dim (N of the MMA)
constexpr uint32_t kBox = 128 * 128;            // one 128-row x 64-col bf16 TMA box = 16 KiB
constexpr uint32_t kQOff = 0;                   // Q tile: [k-half 0..1] boxes
constexpr uint32_t kCOff = 2 * kBox;            // C tile: same
constexpr uint32_t kHOff = 4 * kBox;            // dH stages: [stage][head of pair] boxes
// Kernel modes: 0 the plain score branch; 1 the normalised branch with the key rows rescaled in shared
// memory by a fourth warpgroup; 2 the normalised branch reading keys and queries prepared in scratch
// (k_norm_prep: the key rows r (.) dH rounded once to fp16, the Q rows scaled to fp16 and their factors).
// Shared-memory layout per mode: modes 0-1 keep a 3-stage ring of [dH_h | dH_h+1] and two staging tiles
// per softmax warp (the two column halves of its R rows leave through them without waiting for each other,
// and tile 0 also brings in the next pair's E rows); mode 2 stages [dH_h | dH_h+1 | K_h | K_h+1] in a
// 2-stage ring and gives each softmax warp one tile (R's two halves leave through it one after the other).
template <int kMode> struct SmaLayout {
    static constexpr int kStg = kMode == 2 ? 2 : kStages;
    static constexpr uint32_t kStageBytes = (kMode == 2 ? 4 : 2) * kBox;
    static constexpr uint32_t kTileBytes = kMode == 2 ? 4096 : 8192;  // per softmax warp
    static constexpr uint32_t kStgOff = kHOff + kStg * kStageBytes;
    static constexpr uint32_t kBarOff = kStgOff + 8 * kTileBytes;
    static constexpr uint32_t kQfacOff = kBarOff + 256;            // mode 1: per-row Q factors (128 floats)
    static constexpr uint32_t kSmemBytes = kQfacOff + 512 + 1024;  // + alignment slack
    static_assert(kSmemBytes <= 232448, "SMA kernel exceeds the shared memory of a CTA");
};
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// (d0, d1) += (a0 b0, a1 b1): two fp32 FMAs, each rounded to nearest, in one packed instruction (sm_100
// executes fma.rn.f32x2 at twice the scalar FMA rate)
__device__ __forceinline__ void fma2(float &d0, float &d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%0, %1};\n\t"
        "fma.rn.f32x2 rc, ra, rb, rc;\n\tmov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O and d may grow by at most 2^8 before rescaling

enum { BAR_QC_FULL = 0, BAR_QC_EMPTY, BAR_MMA_DONE, BAR_STAGE_FULL, BAR_STAGE_EMPTY = BAR_STAGE_FULL + kStages,
       BAR_TMEM_FULL = BAR_STAGE_EMPTY + kStages, BAR_TMEM_EMPTY = BAR_TMEM_FULL + 2, BAR_E_FULL = BAR_TMEM_EMPTY + 2,
       BAR_C_DONE = BAR_E_FULL + 8, BAR_SCALED = BAR_C_DONE + kStages, BAR_Q_READY = BAR_SCALED + kStages,
       BAR_MMA_DONE2 = BAR_Q_READY + 1, BAR_COUNT };
static_assert(BAR_COUNT * 8 + 8 <= 256, "barrier block overflows its 256 bytes");

struct SmaTcParams {
    Shape s;
    int hpi;      // heads per work item (even, divides H / G)
    int ntiles;      // 128-token tiles per chunk (S >= 128); 1 when tiles span chunks
    int64_t nslots;  // S < 128: tiles per batch row, ceil(L / 128)
    int ngh;      // head groups per batch row = H / hpi
    int64_t n_items;
    const __nv_bfloat16 *E;
    float *out;   // R; with combine, out (holding Y on entry), to which g R is added
    float *lse;
    const float *g;
    int64_t g_sb, g_st, g_sh;
    int combine;
    float norm_eps;  // normalised score branch: the epsilon inside every RMS
    int hpe;         // heads per E group (1: E per head)
    // mode 2: the part of RMSNorm(Q_t) left out of the fp16 Q rows, [Bt, L, G]
    const float *qfac;
};

// A work item is one 128-token tile and one head group, longest first. With S a multiple of 128
// (kMultiChunk false) the tile is the tile-th of chunk i and takes the chunk steps j < i; the order is
// (chunk i descending, batch row, tile of the chunk, head group), so the tiles of a chunk, which read the
// same chunk memories, run side by side, and a tile past the end of a ragged last chunk has no rows.
// With S < 128 (kMultiChunk, S dividing 128) i is the tile's index in its row and the tile spans 128 / S
// chunks: it takes the steps below its last row's chunk, and each row skips the steps at or after its
// own chunk. Item counts stay below 2^31 (checked on the host): the decode runs in 32-bit arithmetic.
struct Item {
    int64_t i, b, tile, hg;
};

template <bool kMultiChunk>
__device__ __forceinline__ Item decode_item(const SmaTcParams &p, int64_t k) {
    const uint32_t ngh = (uint32_t)p.ngh, per_b = (uint32_t)p.ntiles * ngh, per_i = (uint32_t)p.s.Bt * per_b;
    const uint32_t k32 = (uint32_t)k;
    Item it;
    const uint32_t q = k32 / per_i;
    if constexpr (kMultiChunk)
        it.i = p.nslots - 1 - (int64_t)q;
    else
        it.i = p.s.M - 1 - (int64_t)q;  // longest items (latest target chunks) first
    uint32_t r = k32 - q * per_i;
    const uint32_t b = r / per_b;
    r -= b * per_b;
    const uint32_t tile = r / ngh;
    it.b = b;
    it.tile = tile;
    it.hg = r - tile * ngh;
    return it;
}

template <bool kMultiChunk>
__device__ __forceinline__ int tile_rows(const SmaTcParams &p, const Item &it) {
    if constexpr (kMultiChunk) {
        return (int)min((int64_t)kTileRows, p.s.L - it.i * kTileRows);
    } else {
        const int64_t t0 = it.i * p.s.S + it.tile * kTileRows;
        const int64_t end = min(p.s.L, (it.i + 1) * p.s.S);
        return (int)max((int64_t)0, min((int64_t)kTileRows, end - t0));
    }
}

// chunk steps of a multi-chunk tile: the chunk of its last row
__device__ __forceinline__ int64_t multi_steps(const SmaTcParams &p, const Item &it) {
    return (it.i * kTileRows + min((int64_t)kTileRows, p.s.L - it.i * kTileRows) - 1) / p.s.S;
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// TMA coordinates of the 32 E rows (this warp's tokens) of head (hg * hpi + hp + e) in item k; false when
// the pair reads no E (k past the last item, an item without history, an empty tile).
template <bool kMultiChunk>
__device__ __forceinline__ bool e_coords(const SmaTcParams &p, int64_t k, int hp, int e, int quarter, int32_t &x,
                                         int32_t &y, int32_t &z) {
    if (k >= p.n_items) return false;
    const Item it = decode_item<kMultiChunk>(p, k);
    if constexpr (kMultiChunk) {
        if (multi_steps(p, it) == 0) return false;
    } else {
        if (it.i == 0 || tile_rows<false>(p, it) == 0) return false;
    }
    x = (int32_t)((((int)it.hg * p.hpi + hp + e) / p.hpe) * kP);  // E group of the head
    y = (int32_t)((kMultiChunk ? it.i * kTileRows : it.i * p.s.S + it.tile * kTileRows) + quarter * 32);
    z = (int32_t)it.b;
    return true;
}

template <bool kMultiChunk, int kMode>
__global__ void __launch_bounds__(kMode == 1 ? kTcThreadsNorm : kTcThreads, 1)
    k_sma_fwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC,
                 const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmE,
                 const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmK,
                 const SmaTcParams p) {
    constexpr bool kNorm = kMode == 1;     // the key rows are rescaled in place by the scaler warpgroup
    constexpr bool kNormAny = kMode != 0;  // the normalised score branch (App. B.1)
    using Lay = SmaLayout<kMode>;
    constexpr int kStg = Lay::kStg;
    constexpr uint32_t kBarOff = Lay::kBarOff, kStgOff = Lay::kStgOff, kQfacOff = Lay::kQfacOff;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kBarOff);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kBarOff + BAR_COUNT * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kBarOff + BAR_COUNT * 8 + 4);
    auto bar = [&](int k) { return smem_u32(&bars[k]); };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(bar(BAR_QC_FULL), 1);
        // normalised branch: the softmax warps also read the item's Q row factors before the tile is reused
        // modes 0 and 2: both MMA issuers commit when their MMAs of an item are done
        mbar_init(bar(BAR_QC_EMPTY), kNorm ? 9 : 2);
        mbar_init(bar(BAR_MMA_DONE), 1);
        mbar_init(bar(BAR_MMA_DONE2), 1);
        for (int s = 0; s < kStg; ++s) {
            mbar_init(bar(BAR_STAGE_FULL + s), 1);
            mbar_init(bar(BAR_STAGE_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(BAR_TMEM_FULL + b), 1);
            mbar_init(bar(BAR_TMEM_EMPTY + b), 8);  // one arrival per softmax warp
        }
        for (int w = 0; w < 8; ++w) mbar_init(bar(BAR_E_FULL + w), 1);  // one per softmax warp
        if constexpr (kNorm) {
            for (int s = 0; s < kStages; ++s) {
                mbar_init(bar(BAR_C_DONE + s), 1);  // the C chain has read the stage
                mbar_init(bar(BAR_SCALED + s), 4);  // the four scaler warps have rescaled its rows
            }
            mbar_init(bar(BAR_Q_READY), 4);  // the four scaler warps have rescaled the item's Q tile
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmH);
        tma_prefetch_desc(&tmR);
        tma_prefetch_desc(&tmE);
        if constexpr (kMode == 2) tma_prefetch_desc(&tmK);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int *err = &g_dart_ctl.err;
    const Shape &s = p.s;

    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        setmaxnreg_dec<kNorm ? kRegsLowNorm : kRegsLow>();
        if (lane == 0) {
            uint32_t qc_uses = 0;
            int st = 0;            // ring slot of the next load
            uint32_t ph = 0;       // parity of the ring's current pass
            int last_ph[kStg];  // parity of the last load into each slot (-1: none)
            for (int q = 0; q < kStg; ++q) last_ph[q] = -1;
            bool qc_loaded = false;
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const Item it = decode_item<kMultiChunk>(p, k);
                if constexpr (kMultiChunk) {
                    if (multi_steps(p, it) == 0) continue;
                } else {
                    if (it.i == 0 || tile_rows<false>(p, it) == 0) continue;
                }
                const int64_t nsteps = kMultiChunk ? multi_steps(p, it) : it.i;
                const int64_t h0 = it.hg * p.hpi;
                const int64_t grp = h0 / (s.H / s.G);
                if (!mbar_wait(bar(BAR_QC_EMPTY), (qc_uses & 1) ^ 1, abort_flag, err, 11)) goto producer_end;
                mbar_arrive_expect_tx(bar(BAR_QC_FULL), 4 * kBox);
                {
                    const int32_t y =
                        (int32_t)(it.b * s.L + (kMultiChunk ? it.i * kTileRows : it.i * s.S + it.tile * kTileRows));
                    for (int kh = 0; kh < 2; ++kh) {
                        const int32_t x = (int32_t)(grp * kN + kh * 64);
                        tma_load_2d(sbase + kQOff + kh * kBox, &tmQ, x, y, bar(BAR_QC_FULL));
                        tma_load_2d(sbase + kCOff + kh * kBox, &tmC, x, y, bar(BAR_QC_FULL));
                    }
                }
                ++qc_uses;
                qc_loaded = true;
                for (int hp = 0; hp < p.hpi; hp += 2) {
                    for (int64_t j = 0; j < nsteps; ++j) {
                        if (!mbar_wait(bar(BAR_STAGE_EMPTY + st), ph ^ 1, abort_flag, err, 12)) goto producer_end;
                        mbar_arrive_expect_tx(bar(BAR_STAGE_FULL + st), Lay::kStageBytes);
                        for (int e = 0; e < 2; ++e) {
                            const int32_t y = (int32_t)(((it.b * s.H + h0 + hp + e) * s.M + j) * kN);
                            const uint32_t slot = sbase + kHOff + st * Lay::kStageBytes;
                            tma_load_2d(slot + e * kBox, &tmH, 0, y, bar(BAR_STAGE_FULL + st));
                            if constexpr (kMode == 2)  // the prepared fp16 key rows beside the stored memories
                                tma_load_2d(slot + (2 + e) * kBox, &tmK, 0, y, bar(BAR_STAGE_FULL + st));
                        }
                        last_ph[st] = (int)ph;
                        if (++st == kStg) {
                            st = 0;
                            ph ^= 1;
                        }
                    }
                }
            }
        producer_end:
            // never leave a copy in flight into shared memory that is about to be released
            for (int q = 0; q < kStg; ++q)
                if (last_ph[q] >= 0) mbar_drain(bar(BAR_STAGE_FULL + q), (uint32_t)last_ph[q]);
            if (qc_loaded) mbar_drain(bar(BAR_QC_FULL), (qc_uses - 1) & 1);
        }
    } else if (warp == 1 || (!kNorm && warp == 2)) {
        // -------------------------------- MMA ---------------------------------
        // Modes 0 and 2: two issuers, lane 0 of warps 1 and 2, take alternate chunk steps (issuer i the
        // steps of accumulator buffer i). A step's 16 MMAs take about as long to issue as to run, so
        // with one issuer the tensor pipe ran dry while that thread committed and checked the next step's
        // barriers; with two, one issues while the other does that.
        setmaxnreg_dec<kNorm ? kRegsLowNorm : kRegsLow>();
        constexpr int kIssuers = kNorm ? 1 : 2;
        const int issuer = warp - 1;
        if (lane == 0) {
            // M=128 tokens, N=128 = two heads' 64 value columns, A K-major, B MN-major (two
            // 64-column blocks, the second head's box 16 KiB after the first)
            constexpr uint32_t idesc = idesc_bf16_f32(kTileRows, 2 * kP, false, true);
            const uint64_t qdesc0 = smem_desc_sw128(sbase + kQOff, 16, 1024);
            const uint64_t cdesc0 = smem_desc_sw128(sbase + kCOff, 16, 1024);
            uint32_t qc_uses = 0, tb = 0;
            int st = 0;       // ring slot of the next stage
            uint32_t ph = 0;  // parity of the ring's current pass
            bool issued = false;
            // normalised branch: the Q chain of a stage waits for its rows to be rescaled, so it is issued
            // one step late, after the next stage's C chain (pst: its stage, -1 for none)
            // Its operands are fp16: the Q tile scaled by a power of two per row and the rescaled key rows.
            int pst = -1, pbuf = 0;
            uint32_t pph = 0;
            bool q_wait = false;  // the item's Q tile is still being rescaled
            constexpr uint32_t idesc_h = idesc_f32acc(kTileRows, 2 * kP, false, true, true);
            auto issue_q = [&]() -> bool {
                if (q_wait) {
                    if (!mbar_wait(bar(BAR_Q_READY), (qc_uses - 1) & 1, abort_flag, err, 25)) return false;
                    q_wait = false;
                }
                if (!mbar_wait(bar(BAR_SCALED + pst), pph, abort_flag, err, 24)) return false;
                tc_fence_after();
                const uint64_t bd0 = smem_desc_sw128(sbase + kHOff + pst * Lay::kStageBytes, kBox, 1024);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t aoff = (uint64_t)((((kk >> 2) * kBox) + (kk & 3) * 32) >> 4);
                    mma_bf16(tmem + pbuf * 256, qdesc0 + aoff, bd0 + (uint64_t)((kk * 2048) >> 4), idesc_h, kk > 0);
                }
                mma_commit(bar(BAR_STAGE_EMPTY + pst));
                mma_commit(bar(BAR_TMEM_FULL + pbuf));
                pst = -1;
                return true;
            };
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const Item it = decode_item<kMultiChunk>(p, k);
                if constexpr (kMultiChunk) {
                    if (multi_steps(p, it) == 0) continue;
                } else {
                    if (it.i == 0 || tile_rows<false>(p, it) == 0) continue;
                }
                const int64_t nsteps = kMultiChunk ? multi_steps(p, it) : it.i;
                if (!mbar_wait(bar(BAR_QC_FULL), qc_uses & 1, abort_flag, err, 21)) goto mma_end;
                ++qc_uses;
                if constexpr (kNorm) q_wait = true;
                tc_fence_after();
                for (int hp = 0; hp < p.hpi; hp += 2) {
                    for (int64_t j = 0; j < nsteps; ++j) {
                        if (kIssuers == 2 && (int)(tb & 1) != issuer) {  // the other issuer's step
                            if (++st == kStg) {
                                st = 0;
                                ph ^= 1;
                            }
                            ++tb;
                            continue;
                        }
                        if (!mbar_wait(bar(BAR_STAGE_FULL + st), ph, abort_flag, err, 22)) goto mma_end;
                        const int buf = tb & 1;
                        if (!mbar_wait(bar(BAR_TMEM_EMPTY + buf), ((tb >> 1) & 1) ^ 1, abort_flag, err, 23))
                            goto mma_end;
                        tc_fence_after();
                        const uint64_t bdesc0 = smem_desc_sw128(sbase + kHOff + st * Lay::kStageBytes, kBox, 1024);
                        const uint32_t dq = tmem + buf * 256;
                        if constexpr (kMode == 2) {
                            // values C dH[j] (bf16) and keys Q16 K[j] (fp16: the prepared Q rows against the
                            // prepared key rows, two boxes after the stored memories)
                            const uint64_t kdesc0 = bdesc0 + (uint64_t)((2 * kBox) >> 4);
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint64_t aoff = (uint64_t)((((kk >> 2) * kBox) + (kk & 3) * 32) >> 4);
                                const uint64_t boff = (uint64_t)((kk * 2048) >> 4);
                                mma_bf16(dq, qdesc0 + aoff, kdesc0 + boff, idesc_h, kk > 0);
                                mma_bf16(dq + 128, cdesc0 + aoff, bdesc0 + boff, idesc, kk > 0);
                            }
                            mma_commit(bar(BAR_STAGE_EMPTY + st));
                            mma_commit(bar(BAR_TMEM_FULL + buf));
                            issued = true;
                        } else if constexpr (kNorm) {
                            // values C dH[j] from the stage as loaded; the keys wait for the rescaled rows
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint64_t aoff = (uint64_t)((((kk >> 2) * kBox) + (kk & 3) * 32) >> 4);
                                mma_bf16(dq + 128, cdesc0 + aoff, bdesc0 + (uint64_t)((kk * 2048) >> 4), idesc,
                                         kk > 0);
                            }
                            mma_commit(bar(BAR_C_DONE + st));
                            issued = true;
                            if (pst >= 0 && !issue_q()) goto mma_end;
                            pst = st;
                            pph = ph;
                            pbuf = buf;
                        } else {
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint64_t aoff = (uint64_t)((((kk >> 2) * kBox) + (kk & 3) * 32) >> 4);
                                const uint64_t bdesc = bdesc0 + (uint64_t)((kk * 2048) >> 4);
                                mma_bf16(dq, qdesc0 + aoff, bdesc, idesc, kk > 0);
                                mma_bf16(dq + 128, cdesc0 + aoff, bdesc, idesc, kk > 0);
                            }
                            mma_commit(bar(BAR_STAGE_EMPTY + st));
                            mma_commit(bar(BAR_TMEM_FULL + buf));
                            issued = true;
                        }
                        if (++st == kStg) {
                            st = 0;
                            ph ^= 1;
                        }
                        ++tb;
                    }
                }
                if constexpr (kNorm) {  // the item's last Q chain reads the Q tile: issue it before release
                    if (pst >= 0 && !issue_q()) goto mma_end;
                }
                mma_commit(bar(BAR_QC_EMPTY));
            }
        mma_end:
            if (issued) {  // wait until every issued MMA has finished before tensor memory is released
                const uint32_t done = bar(issuer ? BAR_MMA_DONE2 : BAR_MMA_DONE);
                mma_commit(done);
                mbar_drain(done, 0);
            }
        }
    } else if (warp < 4) {
        setmaxnreg_dec<kNorm ? kRegsLowNorm : kRegsLow>();  // no role, registers only
    } else if (kNorm && warp >= 12) {
        setmaxnreg_dec<kRegsScaler>();
        if constexpr (kNorm) {
            // ------------------------- key-side row scaler -------------------------
            // Normalised score branch (App. B.1 eq 26): the key of chunk j is r_j (.) (dH[j] E_t) with
            // r_{j,n} = (mean_p dH[j]_{n,p}^2 + eps)^(-1/2), i.e. the Q chain reads diag(r_j) dH[j]. Once the
            // C chain has read a stage, warps 12 and 14 rescale the rows of the pair's first head in place, to
            // fp16, and warps 13 and 15 those of the second, each warp half the rows, each lane two (one
            // warp on each of the SM's four schedulers, which the softmax warps share). A row is 128
            // contiguous bytes (the 128-byte swizzle only permutes its 16-byte pieces), read starting at a
            // lane-dependent piece so that the eight lanes of a shared-memory phase hit different banks.
            // fp16 (11 significant bits; the rescaled rows have unit RMS, so no range is lost) rather than
            // bf16: the normalised logits spread over several units, and a bf16 rounding of the keys moved
            // the softmax weights by more than the bf16 tolerance allows.
            const int sw = warp - 12, e = sw & 1, rh = sw >> 1;
            int st = 0;
            uint32_t ph = 0, qc_uses = 0;
            float *qfac = reinterpret_cast<float *>(sm + kQfacOff);
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const Item it = decode_item<kMultiChunk>(p, k);
                if constexpr (kMultiChunk) {
                    if (multi_steps(p, it) == 0) continue;
                } else {
                    if (it.i == 0 || tile_rows<false>(p, it) == 0) continue;
                }
                const int64_t nsteps = kMultiChunk ? multi_steps(p, it) : it.i;
                // The item's Q tile to fp16, row t scaled by sc_t = 2^k_t, the power of two at or below
                // (mean_n Q_t^2 + eps)^(-1/2): the scaled row is exact in fp16 (8 significant bits, largest
                // element at most sqrt(N)), and the rest of RMSNorm(Q_t), inv_q / sc_t, goes to the softmax
                // warps through qfac. Each lane takes one row.
                if (!mbar_wait(bar(BAR_QC_FULL), qc_uses & 1, abort_flag, err, 42)) goto scaler_end;
                ++qc_uses;
                {
                    const int t = sw * 32 + lane;
                    float sq0 = 0.f, sq1 = 0.f;
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(sm + kQOff + kh * kBox + t * 128 +
                                                                             ((q ^ (lane & 7)) << 4));
                            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const float lo = __uint_as_float(w[u] << 16), hi = __uint_as_float(w[u] & 0xffff0000u);
                                sq0 = fmaf(lo, lo, sq0);
                                sq1 = fmaf(hi, hi, sq1);
                            }
                        }
                    }
                    const float inv_q = rsqrtf((sq0 + sq1) * (1.f / kN) + p.norm_eps);
                    const float sc = __uint_as_float(__float_as_uint(inv_q) & 0x7f800000u);
                    qfac[t] = inv_q / sc;
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            uint8_t *ptr = sm + kQOff + kh * kBox + t * 128 + ((q ^ (lane & 7)) << 4);
                            const uint4 v = *reinterpret_cast<const uint4 *>(ptr);
                            uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const __half2 h2 = __floats2half2_rn(__uint_as_float(w[u] << 16) * sc,
                                                                     __uint_as_float(w[u] & 0xffff0000u) * sc);
                                w[u] = *reinterpret_cast<const uint32_t *>(&h2);
                            }
                            *reinterpret_cast<uint4 *>(ptr) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BAR_Q_READY));
                for (int hp = 0; hp < p.hpi; hp += 2) {
                    for (int64_t j = 0; j < nsteps; ++j) {
                        if (!mbar_wait(bar(BAR_C_DONE + st), ph, abort_flag, err, 41)) goto scaler_end;
                        tc_fence_after();
                        uint8_t *box = sm + kHOff + (st * 2 + e) * kBox;
#pragma unroll 1
                        for (int r = 0; r < 2; ++r) {
                            uint8_t *rowp = box + (rh * 64 + lane + 32 * r) * 128;
                            float rr;
                            {
                                float sq0 = 0.f, sq1 = 0.f;  // first pass: the row's sum of squares
#pragma unroll
                                for (int q = 0; q < 8; ++q) {
                                    const uint4 v = *reinterpret_cast<const uint4 *>(rowp + ((q ^ (lane & 7)) << 4));
                                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                                    for (int u = 0; u < 4; ++u) {
                                        const float lo = __uint_as_float(w[u] << 16),
                                                    hi = __uint_as_float(w[u] & 0xffff0000u);
                                        sq0 = fmaf(lo, lo, sq0);
                                        sq1 = fmaf(hi, hi, sq1);
                                    }
                                }
                                rr = rsqrtf((sq0 + sq1) * (1.f / kP) + p.norm_eps);
                            }
#pragma unroll
                            for (int q = 0; q < 8; ++q) {  // second pass: rescale in place
                                const uint4 v = *reinterpret_cast<const uint4 *>(rowp + ((q ^ (lane & 7)) << 4));
                                uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    const __half2 h2 = __floats2half2_rn(__uint_as_float(w[u] << 16) * rr,
                                                                         __uint_as_float(w[u] & 0xffff0000u) * rr);
                                    w[u] = *reinterpret_cast<const uint32_t *>(&h2);
                                }
                                *reinterpret_cast<uint4 *>(rowp + ((q ^ (lane & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                            }
                        }
                        fence_async_smem();  // the rescaled rows, written by the generic proxy, feed the MMA
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(BAR_SCALED + st));
                        if (++st == kStages) {
                            st = 0;
                            ph ^= 1;
                        }
                    }
                }
            }
        scaler_end:;
        }
    } else {
        // ------------------------------ softmax -------------------------------
        setmaxnreg_inc<kNorm ? kRegsHighNorm : kRegsHigh>();
        const int e = (warp - 4) >> 2;      // warpgroup = head of the pair
        const int quarter = warp & 3;       // tensor-memory lane quarter this warp may access
        const int row = quarter * 32 + lane;
        const float escale = kLog2e * rsqrtf((float)kN);
        uint32_t tb = 0;
        // This warp's 4 KiB tiles: tile 0 carries, in turn, the E rows of the next pair (TMA load,
        // issued one chunk into the current pair) and the first column half of the current pair's R
        // rows (TMA store at its end); tile 1 the second half (mode 2, with one tile: tile 0 again, once
        // the first half's store has read it).
        uint8_t *stg = sm + kStgOff + (warp - 4) * Lay::kTileBytes;
        const uint32_t ebar = bar(BAR_E_FULL + (warp - 4));
        // E_t of the current pair: unpacked to fp32 once per pair (modes 0 and 2), so that the per-step logit
        // loop does no unpacking; as bf16 pairs in mode 1, whose warps have fewer registers
        float ef[kP];
        uint32_t ev[kP / 2];
        int64_t ev_k = -1, pend_k = -1;  // pair whose E is in ev / in flight into the tile
        int ev_hp = 0, pend_hp = 0;
        uint32_t e_uses = 0;
        uint32_t qc_uses = 0;  // normalised branch: items whose Q row factor was read
        float inv_q = 1.f;     // normalised branch: the part of RMSNorm(Q_t) left out of the fp16 Q tile
        // E rows of pair (k2, hp2) into the tile, once its previous R stores have read it
        auto issue_e = [&](int64_t k2, int hp2) {
            int32_t x, y, z;
            if (!e_coords<kMultiChunk>(p, k2, hp2, e, quarter, x, y, z)) return;
            __syncwarp();  // every lane is done with the tile's previous contents
            if (lane == 0) {
                bulk_wait_group_read<0>();
                fence_async_smem();
                mbar_arrive_expect_tx(ebar, 4096);
                tma_load_3d(smem_u32(stg), &tmE, x, y, z, ebar);
            }
            pend_k = k2;
            pend_hp = hp2;
        };
        // the pending E rows into ev; false when the wait gave up
        auto take_e = [&]() -> bool {
            if (!mbar_wait(ebar, e_uses & 1, abort_flag, err, 32)) return false;
            ++e_uses;
            const uint8_t *srow = stg + lane * 128;
#pragma unroll
            for (int q = 0; q < kP / 8; ++q) {
                const uint4 v = *reinterpret_cast<const uint4 *>(srow + ((q ^ (lane & 7)) << 4));
                if constexpr (kMode == 1) {
                    ev[4 * q] = v.x;
                    ev[4 * q + 1] = v.y;
                    ev[4 * q + 2] = v.z;
                    ev[4 * q + 3] = v.w;
                } else {
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        ef[8 * q + 2 * i] = __uint_as_float(w4[i] << 16);
                        ef[8 * q + 2 * i + 1] = __uint_as_float(w4[i] & 0xffff0000u);
                    }
                }
            }
            __syncwarp();
            ev_k = pend_k;
            ev_hp = pend_hp;
            pend_k = -1;
            return true;
        };
        for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
            const Item it = decode_item<kMultiChunk>(p, k);
            const int rows = tile_rows<kMultiChunk>(p, it);
            if (rows == 0) continue;
            const int64_t t = (kMultiChunk ? it.i * kTileRows : it.i * s.S + it.tile * kTileRows) + row;
            int64_t nsteps = it.i, my_chunk = 0;  // multi-chunk tiles: steps of the tile, chunk of this row
            if constexpr (kMultiChunk) {
                nsteps = multi_steps(p, it);
                my_chunk = t / s.S;
            }
            const bool valid = row < rows;
            if constexpr (kMode == 2) {
                // RMSNorm of Q_t (App. B.1 eq 25): the prepared fp16 Q rows hold all of it but this factor
                if (nsteps > 0 && valid) inv_q = __ldg(p.qfac + (it.b * s.L + t) * s.G + (it.hg * p.hpi) / (s.H / s.G));
            }
            if constexpr (kNorm) {
                // RMSNorm of Q_t (App. B.1 eq 25): the scaler warps put all of it but a factor into the fp16
                // Q tile; that factor enters the logit scale. Reading it frees the tile for the next item.
                if (nsteps > 0) {
                    if (!mbar_wait(bar(BAR_Q_READY), qc_uses & 1, abort_flag, err, 33)) goto softmax_end;
                    ++qc_uses;
                    inv_q = reinterpret_cast<const float *>(sm + kQfacOff)[row];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(BAR_QC_EMPTY));
                }
            }
            for (int hp = 0; hp < p.hpi; hp += 2) {
                const int64_t h = it.hg * p.hpi + hp + e;
                if (nsteps == 0) {  // no historical chunk for any row of the tile
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
                float esc = escale;  // logit scale; the normalised branch folds RMSNorm of Q_t and E_t into it
                if constexpr (kNormAny) {
                    float se0 = 0.f, se1 = 0.f;
#pragma unroll
                    for (int q = 0; q < kP / 2; ++q) {
                        const float lo = kMode == 1 ? __uint_as_float(ev[q] << 16) : ef[2 * q];
                        const float hi = kMode == 1 ? __uint_as_float(ev[q] & 0xffff0000u) : ef[2 * q + 1];
                        se0 = fmaf(lo, lo, se0);
                        se1 = fmaf(hi, hi, se1);
                    }
                    esc = escale * inv_q * rsqrtf((se0 + se1) * (1.f / kP) + p.norm_eps);
                }
                // fused layer: this row's gate, fetched before the chunk loop
                const float gate = (p.combine && valid) ? __ldg(p.g + it.b * p.g_sb + t * p.g_st + h * p.g_sh) : 0.f;
                int64_t nk = k;  // the next pair
                int nhp = hp + 2;
                if (nhp >= p.hpi) {
                    nhp = 0;
                    nk = sched_next(k);
                }
                float O[kP];
#pragma unroll
                for (int q = 0; q < kP; ++q) O[q] = 0.f;
                float m = -INFINITY, d = 0.f;
                for (int64_t j = 0; j < nsteps; ++j) {
                    const int buf = tb & 1;
                    if (!mbar_wait(bar(BAR_TMEM_FULL + buf), (tb >> 1) & 1, abort_flag, err, 31)) goto softmax_end;
                    tc_fence_after();
                    const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + buf * 256 + e * kP;
                    // logit: (Q_t dH[j]) . E_t, read in two 32-column halves, four partial sums (two packed pairs)
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float u[32];
                        tmem_ld_32x32b_x32_after(ta + half * 32, u, acc[0]);
                        tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            float lo, hi;
                            if constexpr (kMode == 1) {
                                const uint32_t w = ev[16 * half + q];
                                lo = __uint_as_float(w << 16);
                                hi = __uint_as_float(w & 0xffff0000u);
                            } else {
                                lo = ef[32 * half + 2 * q];
                                hi = ef[32 * half + 2 * q + 1];
                            }
                            fma2(acc[2 * (q & 1)], acc[2 * (q & 1) + 1], u[2 * q], u[2 * q + 1], lo, hi);
                        }
                    }
                    float l2 = ((acc[0] + acc[1]) + (acc[2] + acc[3])) * (kNormAny ? esc : escale);  // l_{t,j}, log2 units
                    float pw;
                    if constexpr (kMultiChunk) {  // a row takes no part in the steps at or after its chunk
                        const bool live = j < my_chunk;
                        if (live && l2 > m + kRescaleThreshold) {
                            const float f = exp2f(m - l2);
                            d *= f;
#pragma unroll
                            for (int q = 0; q < kP; ++q) O[q] *= f;
                            m = l2;
                        }
                        __syncwarp();  // reconverge before the warp-collective tensor-memory loads
                        pw = live ? exp2f(l2 - m) : 0.f;
                    } else {
                        if (l2 > m + kRescaleThreshold) {  // lazy rescale: only when the running max grows a lot
                            const float f = exp2f(m - l2);
                            d *= f;
#pragma unroll
                            for (int q = 0; q < kP; ++q) O[q] *= f;
                            m = l2;
                        }
                        __syncwarp();  // reconverge before the warp-collective tensor-memory loads
                        pw = exp2f(l2 - m);
                    }
                    d += pw;
                    // value C_t dH[j], accumulated with weight pw
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float v[32];
                        tmem_ld_32x32b_x32_after(ta + 128 + half * 32, v, pw + O[32 * half]);
                        tmem_ld_wait();
                        if (half == 1) {  // both halves read: hand the buffer back to the MMA early
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(bar(BAR_TMEM_EMPTY + buf));
                        }
#pragma unroll
                        for (int q = 0; q < 32; q += 2)
                            fma2(O[32 * half + q], O[32 * half + q + 1], pw, pw, v[q], v[q + 1]);
                    }
                    ++tb;
                    if (j == 0) issue_e(nk, nhp);  // a chunk in, the previous pair's R stores are done
                }
                // the next pair's E rows out of the tile before R goes through it
                if (pend_k >= 0 && !take_e()) goto softmax_end;
                // d = 0 only for a row without history in a multi-chunk tile: R = 0 there
                const float inv = (!kMultiChunk || d > 0.f) ? 1.f / d : 0.f;
                {
                    // R = O / d through this warp's staging tiles, 32 rows x 32 columns each, by TMA store; in
                    // the fused layer (combine) g R instead, added into out (which holds Y) by a TMA
                    // reduction, eq (11). Either way rows past the end of the batch row are clipped.
                    const float sc = p.combine ? gate * inv : inv;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        // the tiles' previous users (the last pair's stores, the E load) are done: E was
                        // taken above, and the stores had a whole pair to read them; with one tile the
                        // second half waits for the first half's store to have read it
                        if ((half == 0 || kMode == 2) && lane == 0) bulk_wait_group_read<0>();
                        __syncwarp();
                        uint8_t *tile = stg + (kMode == 2 ? 0 : half * 4096);
                        uint8_t *srow = tile + lane * 128;
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            *reinterpret_cast<float4 *>(srow + ((q ^ (lane & 7)) << 4)) =
                                make_float4(O[32 * half + 4 * q] * sc, O[32 * half + 4 * q + 1] * sc,
                                            O[32 * half + 4 * q + 2] * sc, O[32 * half + 4 * q + 3] * sc);
                        fence_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            const int32_t tx = (int32_t)(h * kP + half * 32);
                            const int32_t ty = (int32_t)((kMultiChunk ? it.i * kTileRows
                                                                      : it.i * s.S + it.tile * kTileRows) +
                                                         quarter * 32);
                            if (p.combine)
                                tma_reduce_add_3d(&tmR, smem_u32(tile), tx, ty, (int32_t)it.b);
                            else
                                tma_store_3d(&tmR, smem_u32(tile), tx, ty, (int32_t)it.b);
                            bulk_commit_group();
                        }
                    }
                }
                if (valid && p.lse)
                    p.lse[(it.b * s.H + h) * s.L + t] = (!kMultiChunk || d > 0.f) ? (m + log2f(d)) * kLn2 : -INFINITY;
            }
        }
    softmax_end:
        if (pend_k >= 0) mbar_drain(ebar, e_uses & 1);  // an E load still in flight into the tile
        if (lane == 0) bulk_wait_group<0>();            // every R store has landed before the CTA exits
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

namespace {

}  // namespace

bool tc_shape_ok(const Shape &s, bool bf16) {
    if (!bf16 || s.N != kN || s.P != kP) return false;
    if (s.S % kTileRows != 0 && !(s.S < kTileRows && kTileRows % s.S == 0)) return false;
    if ((s.H / s.G) % 2 != 0) return false;  // two heads of one group per MMA
    if ((s.L + s.S + kTileRows) / kTileRows * s.Bt * (s.H / 2) >= (int64_t(1) << 31)) return false;  // 32-bit decode
    // 32-bit TMA coordinates
    if (s.Bt * s.L >= (int64_t(1) << 31) || s.Bt * s.H * s.M * s.N >= (int64_t(1) << 31)) return false;
    return true;
}

// Operands of the normalised branch (App. B.1 eq 25-26) prepared once per call for mode 2:
//   blocks [0, key_blocks): every chunk memory row n of dH[c], as the key row r_{c,n} dH[c]_n rounded once
//     to fp16, r_{c,n} = (mean_p dH[c]_{n,p}^2 + eps)^(-1/2) (eight lanes a 128-byte row);
//   the other blocks: every row Q_t of a Q/C group, scaled by sc_t = 2^k_t, the power of two at or below
//     iq_t = (mean_n Q_t^2 + eps)^(-1/2), to fp16 (exact: 8 significant bits, largest element at most
//     sqrt(N)), and qfac_t = iq_t / sc_t, the rest of RMSNorm(Q_t), which enters the logit scale (16 lanes
//     a 256-byte row).
__global__ void __launch_bounds__(256) k_norm_prep(const __nv_bfloat16 *__restrict__ dH, const __nv_bfloat16 *__restrict__ Q,
                                                   __half *__restrict__ k16, __half *__restrict__ q16,
                                                   float *__restrict__ qfac, int64_t krows, int64_t qrows,
                                                   int64_t key_blocks, float eps) {
    if (blockIdx.x < key_blocks) {
        const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 3;
        const int part = threadIdx.x & 7;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < krows) v = __ldg(reinterpret_cast<const uint4 *>(dH + row * kP) + part);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float sq = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float lo = __uint_as_float(w[u] << 16), hi = __uint_as_float(w[u] & 0xffff0000u);
            sq = fmaf(lo, lo, fmaf(hi, hi, sq));
        }
        sq += __shfl_xor_sync(0xffffffffu, sq, 4);
        sq += __shfl_xor_sync(0xffffffffu, sq, 2);
        sq += __shfl_xor_sync(0xffffffffu, sq, 1);
        if (row >= krows) return;
        const float r = rsqrtf(sq * (1.f / kP) + eps);
        uint32_t o[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const __half2 h2 = __floats2half2_rn(__uint_as_float(w[u] << 16) * r, __uint_as_float(w[u] & 0xffff0000u) * r);
            o[u] = *reinterpret_cast<const uint32_t *>(&h2);
        }
        reinterpret_cast<uint4 *>(k16 + row * kP)[part] = make_uint4(o[0], o[1], o[2], o[3]);
        return;
    }
    const int64_t row = ((int64_t)(blockIdx.x - key_blocks) * blockDim.x + threadIdx.x) >> 4;
    const int part = threadIdx.x & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row < qrows) v = __ldg(reinterpret_cast<const uint4 *>(Q + row * kN) + part);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float sq = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const float lo = __uint_as_float(w[u] << 16), hi = __uint_as_float(w[u] & 0xffff0000u);
        sq = fmaf(lo, lo, fmaf(hi, hi, sq));
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if (row >= qrows) return;
    const float iq = rsqrtf(sq * (1.f / kN) + eps);
    const float sc = __uint_as_float(__float_as_uint(iq) & 0x7f800000u);
    if (part == 0) qfac[row] = iq / sc;
    uint32_t o[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const __half2 h2 = __floats2half2_rn(__uint_as_float(w[u] << 16) * sc, __uint_as_float(w[u] & 0xffff0000u) * sc);
        o[u] = *reinterpret_cast<const uint32_t *>(&h2);
    }
    reinterpret_cast<uint4 *>(q16 + row * kN)[part] = make_uint4(o[0], o[1], o[2], o[3]);
}

NormPrepWs norm_prep_layout(const Shape &s) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    NormPrepWs w{};
    w.k16 = 0;
    w.q16 = up((size_t)(s.Bt * s.H * s.M * s.N * s.P) * 2);
    w.qfac = w.q16 + up((size_t)(s.Bt * s.L * s.G * s.N) * 2);
    w.total = w.qfac + up((size_t)(s.Bt * s.L * s.G) * 4);
    return w;
}

cudaError_t launch_sma_fwd_tc(const Shape &s, const LayerPtrs &lp, cudaStream_t st) {
    SmaTcParams p{};
    p.s = s;
    const int64_t hpg = s.H / s.G;  // heads sharing one Q/C group
    p.hpi = hpg % 4 == 0 ? 4 : 2;   // heads go in pairs (tc_shape_ok requires H/G even)
    p.ngh = (int)(s.H / p.hpi);
    // S >= 128: every chunk has S / 128 tile slots (some empty past a ragged end); S < 128: one slot per
    // 128 tokens of a row
    p.ntiles = (int)(s.S >= kTileRows ? s.S / kTileRows : 1);
    p.nslots = (s.L + kTileRows - 1) / kTileRows;
    p.n_items = (s.S >= kTileRows ? s.M : p.nslots) * s.Bt * p.ntiles * p.ngh;
    p.E = static_cast<const __nv_bfloat16 *>(lp.E);
    p.combine = lp.combine ? 1 : 0;
    p.out = static_cast<float *>(lp.combine ? lp.Y : lp.R);
    p.lse = lp.lse;
    p.g = lp.g;
    p.g_sb = lp.g_sb;
    p.g_st = lp.g_st;
    p.g_sh = lp.g_sh;
    p.norm_eps = lp.norm_eps;
    const bool prep = lp.score_norm && lp.norm_prep;  // mode 2: the operands prepared in scratch
    const NormPrepWs nw = norm_prep_layout(s);
    uint8_t *nb = static_cast<uint8_t *>(lp.norm_prep);
    p.qfac = prep ? reinterpret_cast<const float *>(nb + nw.qfac) : nullptr;
    p.hpe = (int)heads_per_e(s, lp.e_groups);
    const uint64_t EGP = (uint64_t)(s.H / p.hpe * s.P);  // E row: one P-vector per E group
    CUtensorMap mq, mc, mh, me, mr, mk;
    // the Q rows as loaded: Q itself, or in mode 2 its prepared fp16 rows (2-byte elements either way); mk:
    // the prepared fp16 key rows, laid out as dH (the plain modes pass the dH map, unused)
    const void *qsrc = prep ? static_cast<const void *>(nb + nw.q16) : lp.Q;
    if (!make_tma_map_bf16(&mq, qsrc, (uint64_t)(s.G * s.N), (uint64_t)(s.Bt * s.L), (uint64_t)(s.G * s.N * 2), 64,
                           128) ||
        !make_tma_map_bf16(&mk, prep ? static_cast<const void *>(nb + nw.k16) : lp.dH, (uint64_t)s.P,
                           (uint64_t)(s.Bt * s.H * s.M * s.N), (uint64_t)(s.P * 2), 64, 128) ||
        !make_tma_map_bf16(&mc, lp.C, (uint64_t)(s.G * s.N), (uint64_t)(s.Bt * s.L), (uint64_t)(s.G * s.N * 2), 64,
                           128) ||
        !make_tma_map_bf16(&mh, lp.dH, (uint64_t)s.P, (uint64_t)(s.Bt * s.H * s.M * s.N), (uint64_t)(s.P * 2), 64,
                           128) ||
        !make_tma_map_f32_3d(&mr, p.out, (uint64_t)(s.H * s.P), (uint64_t)s.L, (uint64_t)s.Bt, (uint64_t)(s.H * s.P * 4),
                             (uint64_t)(s.L * s.H * s.P * 4), 32, 32) ||
        !make_tma_map_bf16_3d(&me, lp.E, EGP, (uint64_t)s.L, (uint64_t)s.Bt, EGP * 2, (uint64_t)s.L * EGP * 2, 64, 32))
        return cudaErrorInvalidValue;
    static unsigned long long attr_set = 0;  // per device
    if (!device_flag_set(attr_set)) {
        // the register split of the warpgroups assumes this launch size; a build that gave the kernel
        // fewer registers would leave the softmax warpgroups waiting for registers that do not exist
        struct Fn {
            const void *fn;
            int regs;
            uint32_t smem;
        };
        const Fn fns[] = {
            {reinterpret_cast<const void *>(k_sma_fwd_tc<false, 0>), kRegsLaunch, SmaLayout<0>::kSmemBytes},
            {reinterpret_cast<const void *>(k_sma_fwd_tc<true, 0>), kRegsLaunch, SmaLayout<0>::kSmemBytes},
            {reinterpret_cast<const void *>(k_sma_fwd_tc<false, 1>), kRegsLaunchNorm, SmaLayout<1>::kSmemBytes},
            {reinterpret_cast<const void *>(k_sma_fwd_tc<true, 1>), kRegsLaunchNorm, SmaLayout<1>::kSmemBytes},
            {reinterpret_cast<const void *>(k_sma_fwd_tc<false, 2>), kRegsLaunch, SmaLayout<2>::kSmemBytes},
            {reinterpret_cast<const void *>(k_sma_fwd_tc<true, 2>), kRegsLaunch, SmaLayout<2>::kSmemBytes}};
        for (const auto &f : fns) {
            const void *fn = f.fn;
            cudaFuncAttributes fa{};
            cudaError_t ea = cudaFuncGetAttributes(&fa, fn);
            if (ea != cudaSuccess || fa.numRegs != f.regs) {
                set_last_error("sma_fwd_tc built with an unexpected register count", cudaErrorInvalidConfiguration);
                return ea != cudaSuccess ? ea : cudaErrorInvalidConfiguration;
            }
            cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)f.smem);
            if (e != cudaSuccess) {
                set_last_error("cudaFuncSetAttribute(sma_fwd_tc)", e);
                return e;
            }
        }
        set_device_flag(&attr_set);
    }
    const int64_t grid = std::min<int64_t>(p.n_items, device_sm_count());
    if (prep) {
        const int64_t krows = s.Bt * s.H * s.M * s.N, qrows = s.Bt * s.L * s.G;
        const int64_t kb = (krows * 8 + 255) / 256, qb = (qrows * 16 + 255) / 256;
        launch_begin(KK_KEY_RMS, st);
        k_norm_prep<<<(unsigned)(kb + qb), 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(lp.dH), static_cast<const __nv_bfloat16 *>(lp.Q),
            reinterpret_cast<__half *>(nb + nw.k16), reinterpret_cast<__half *>(nb + nw.q16),
            reinterpret_cast<float *>(nb + nw.qfac), krows, qrows, kb, lp.norm_eps);
        const cudaError_t e = launch_end(KK_KEY_RMS, st);
        if (e != cudaSuccess) return e;
    }
    const int kind = lp.score_norm ? KK_SMA_FWD_NORM_TC : KK_SMA_FWD_TC;
    const bool multi = s.S < kTileRows;
    launch_begin(kind, st);
    if (prep) {
        if (multi)
            k_sma_fwd_tc<true, 2><<<(unsigned)grid, kTcThreads, SmaLayout<2>::kSmemBytes, st>>>(mq, mc, mh, me, mr, mk, p);
        else
            k_sma_fwd_tc<false, 2><<<(unsigned)grid, kTcThreads, SmaLayout<2>::kSmemBytes, st>>>(mq, mc, mh, me, mr, mk, p);
    } else if (lp.score_norm) {
        if (multi)
            k_sma_fwd_tc<true, 1><<<(unsigned)grid, kTcThreadsNorm, SmaLayout<1>::kSmemBytes, st>>>(mq, mc, mh, me, mr, mk,
                                                                                                  p);
        else
            k_sma_fwd_tc<false, 1><<<(unsigned)grid, kTcThreadsNorm, SmaLayout<1>::kSmemBytes, st>>>(mq, mc, mh, me, mr,
                                                                                                   mk, p);
    } else {
        if (multi)
            k_sma_fwd_tc<true, 0><<<(unsigned)grid, kTcThreads, SmaLayout<0>::kSmemBytes, st>>>(mq, mc, mh, me, mr, mk, p);
        else
            k_sma_fwd_tc<false, 0><<<(unsigned)grid, kTcThreads, SmaLayout<0>::kSmemBytes, st>>>(mq, mc, mh, me, mr, mk, p);
    }
    return launch_end(kind, st);
}

int *device_error_word() {
    static int *ptrs[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dart_ctl) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int *>(p);  // DevCtl::err is the block's first member
    }
    return ptrs[dev];
}

int *fp16_range_word() {
    static int *ptrs[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dart_fp16_range) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int *>(p);
    }
    return ptrs[dev];
}

int read_fp16_range(bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dart_fp16_range, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v != 0) {
        int z = 0;
        cudaMemcpyToSymbol(g_dart_fp16_range, &z, sizeof(int));
    }
    return v;
}

int read_device_error(bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dart_ctl, sizeof(int), offsetof(sm100::DevCtl, err)) != cudaSuccess) return -1;
    if (clear && v != 0) {
        int z = 0;
        cudaMemcpyToSymbol(g_dart_ctl, &z, sizeof(int), offsetof(sm100::DevCtl, err));
    }
    return v;
}

cudaError_t set_wait_limit_ns(unsigned long long ns) {
    return cudaMemcpyToSymbol(g_dart_ctl, &ns, sizeof(ns), offsetof(sm100::DevCtl, wait_ns));
}

}  // namespace dart
