// SSD chunk output on tcgen05 (DART paper App. A, eq 19-24; the Mamba-2 chunked
// scan that DART keeps):
//
//   Y_t = sum_{s in c, s <= t} (C_t . B_s) exp(cs_t - cs_s) X_s  +  exp(cs_t) C_t Hprev[c]
//
// Work item = (128-token tile tau of chunk c, batch b, 4 heads). The C tile and
// the chunk's B rows (shared by every head, G = 1) stay in shared memory for the
// item. Per head h and 128-token block sigma <= tau of source tokens:
//   MMA      S = C_tile B_sigma^T                      (M=128 N=128 K=128, fp32 in TMEM)
//   builders P = S o exp(cs_t - cs_s), s <= t          (fp16, written back into the first
//            64 columns of S's own tensor-memory buffer, two values per column)
//            and X_{sigma,h} converted in place bf16 -> fp16 (exact for |x| < 65504)
//   MMA      Y_intra += P X_{sigma,h}                  (A = P from tensor memory, fp16,
//                                                       M=128 N=64 K=128)
// and once per head  Y_inter = C_tile Hprev_h[c]       (M=128 N=64 K=128);
//   epilogue Y = Y_intra + exp(cs_t) Y_inter           (fp32 rows to HBM; in the fused layer the
//            SMA kernel adds g R to them afterwards, eq 11).
// Warps: 0 TMA producer, 1 MMA issuer, 2-9 builders (two groups, one column half of every unit each),
// 10-13 epilogue.
// P is formed in fp16 rather than bf16: the SSD output is heavy-tailed (a few
// dominant terms per row), and a bf16 rounding of P alone costs about 2% of rms(Y).
// This path needs |C_t . B_s| exp(cs_t - cs_s) and |X| below the fp16 range limit (65504); beyond it the
// affected outputs are written as inf or NaN and the kernel raises kRangeSsdOut in the fp16 range word.
#include <cuda.h>
#include <math.h>

#include <algorithm>
#include <type_traits>

#include <cuda_fp16.h>

#include "dart_internal.cuh"
#include "sm100_ptx.cuh"

namespace dart {
namespace {

using namespace sm100;

constexpr int kThreads = 448;  // 14 warps
constexpr int kRows = 128;
constexpr int kN = 128;
constexpr int kP = 64;
constexpr int kHpi = 4;                     // heads per item (divides H / G; else 2 or 1)
constexpr uint32_t kBox = 128 * 128;        // 128 rows x 128 bytes
constexpr int kXSlots = 4;                  // X ring depth (16 KiB per 128-token block)
constexpr uint32_t kCOff = 0;               // C tile: 2 boxes (n 0-63, 64-127)
constexpr uint32_t kBOff = 2 * kBox;        // B blocks: [sigma 0..1][n half] boxes
constexpr uint32_t kHpOff = 6 * kBox;       // Hprev slot (1 box)
constexpr uint32_t kXOff = 7 * kBox;        // X ring
constexpr uint32_t kStgOff = kXOff + kXSlots * kBox;  // epilogue tiles: [epilogue warp][column half] 32 x 128 B
constexpr uint32_t kCsOff = kStgOff + 4 * 8192;       // cs of the item's heads: [item parity][head][256] floats
constexpr uint32_t kBarOff = kCsOff + 2 * kHpi * 256 * 4;
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;
constexpr uint32_t kTmemCols = 512;
// tensor memory: three S/P buffers of 128 columns (three units in flight between the MMA and the builders)
// and one head accumulator [Y_intra 64 | Y_inter 64] at column kYCol
constexpr int kSBufs = 3;
constexpr int kYBufs = 1;
constexpr uint32_t kYCol = kSBufs * 128;
static_assert(kYCol + kYBufs * 128 <= kTmemCols, "tensor memory columns");
constexpr float kLog2e = 1.4426950408889634f;

enum {
    B_ITEM_FULL = 0, B_ITEM_EMPTY, B_HP_FULL, B_HP_EMPTY, B_X_FULL, B_X_EMPTY = B_X_FULL + kXSlots,
    B_S_FULL = B_X_EMPTY + kXSlots, B_S_EMPTY = B_S_FULL + kSBufs, B_P_FULL = B_S_EMPTY + kSBufs,
    B_Y_FULL = B_P_FULL + kSBufs, B_Y_EMPTY = B_Y_FULL + kYBufs, B_MMA_DONE = B_Y_EMPTY + kYBufs, B_GROUP,
    B_COUNT
};

struct SsdTcParams {
    Shape s;
    int hpi, ngh, ntiles;  // heads per item, head groups, 128-token tiles per chunk
    int64_t n_items;
    const float *cs;       // [Bt, H, L]
    float *Y;              // [Bt, L, H, P] fp32
    int *err;
    int *range;            // fp16 range flag word (kRangeSsdOut), or null
};

struct Item {
    int64_t tau, b, c, hg;
};

__device__ __forceinline__ Item decode_item(const SsdTcParams &p, int64_t k) {
    const int64_t per_tau = p.s.Bt * p.s.M * p.ngh;
    Item it;
    it.tau = p.ntiles - 1 - k / per_tau;  // later tiles (more source blocks) first
    int64_t r = k % per_tau;
    it.b = r / (p.s.M * p.ngh);
    r %= p.s.M * p.ngh;
    it.c = r / p.ngh;
    it.hg = r % p.ngh;
    return it;
}

__device__ __forceinline__ int item_rows(const SsdTcParams &p, const Item &it) {
    const int64_t t0 = it.c * p.s.S + it.tau * kRows;
    const int64_t end = min(p.s.L, (it.c + 1) * p.s.S);
    return (int)max((int64_t)0, min((int64_t)kRows, end - t0));
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Two packed bf16 values -> two packed fp16 values (exact for magnitudes in fp16 range).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
    return pack_f16(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__global__ void __launch_bounds__(kThreads, 1)
    k_ssd_out_tc(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmHp,
                 const __grid_constant__ CUtensorMap tmY, const SsdTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kBarOff);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kBarOff + B_COUNT * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kBarOff + B_COUNT * 8 + 4);
    float *cs_sm = reinterpret_cast<float *>(sm + kCsOff);
    auto bar = [&](int k) { return smem_u32(&bars[k]); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape &s = p.s;
    int *err = p.err;

    if (threadIdx.x == 0) {
        for (int k = 0; k < B_COUNT; ++k) {
            uint32_t cnt = 1;
            if (k >= B_Y_EMPTY && k < B_Y_EMPTY + kYBufs) cnt = 4;  // one arrival per epilogue warp
            if (k >= B_P_FULL && k < B_P_FULL + kSBufs) cnt = 8;    // one arrival per builder warp
            if (k == B_GROUP) cnt = 8;  // both builder groups
            mbar_init(bar(k), cnt);
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmHp);
        tma_prefetch_desc(&tmY);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            uint32_t n_items = 0, n_hp = 0, n_x = 0;
            int64_t last_x[kXSlots];
            for (int q = 0; q < kXSlots; ++q) last_x[q] = -1;
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const Item it = decode_item(p, k);
                if (item_rows(p, it) == 0) continue;
                const int64_t h0 = it.hg * p.hpi;
                const int64_t grp = h0 / (s.H / s.G);
                const int nblk = (int)it.tau + 1;
                if (!mbar_wait(bar(B_ITEM_EMPTY), (n_items & 1) ^ 1, abort_flag, err, 41)) goto producer_end;
                mbar_arrive_expect_tx(bar(B_ITEM_FULL), (2 + 2 * nblk) * kBox);
                {
                    const int32_t yt = (int32_t)(it.b * s.L + it.c * s.S + it.tau * kRows);
                    for (int kh = 0; kh < 2; ++kh)
                        tma_load_2d(sbase + kCOff + kh * kBox, &tmC, (int32_t)(grp * kN + kh * 64), yt,
                                    bar(B_ITEM_FULL));
                    for (int sg = 0; sg < nblk; ++sg) {
                        const int32_t ys = (int32_t)(it.b * s.L + it.c * s.S + sg * kRows);
                        for (int kh = 0; kh < 2; ++kh)
                            tma_load_2d(sbase + kBOff + (sg * 2 + kh) * kBox, &tmB, (int32_t)(grp * kN + kh * 64), ys,
                                        bar(B_ITEM_FULL));
                    }
                }
                ++n_items;
                for (int hh = 0; hh < p.hpi; ++hh) {
                    const int64_t h = h0 + hh;
                    // the head's X blocks first: its Hprev waits for the previous head's C Hprev, which the
                    // MMA issues only at that head's first P X
                    for (int sg = 0; sg < nblk; ++sg) {
                        const int slot = n_x % kXSlots;
                        if (!mbar_wait(bar(B_X_EMPTY + slot), ((n_x / kXSlots) & 1) ^ 1, abort_flag, err, 43))
                            goto producer_end;
                        mbar_arrive_expect_tx(bar(B_X_FULL + slot), kBox);
                        tma_load_2d(sbase + kXOff + slot * kBox, &tmX, (int32_t)(h * kP),
                                    (int32_t)(it.b * s.L + it.c * s.S + sg * kRows), bar(B_X_FULL + slot));
                        last_x[slot] = n_x;
                        ++n_x;
                    }
                    if (!mbar_wait(bar(B_HP_EMPTY), (n_hp & 1) ^ 1, abort_flag, err, 42)) goto producer_end;
                    mbar_arrive_expect_tx(bar(B_HP_FULL), kBox);
                    tma_load_2d(sbase + kHpOff, &tmHp, 0, (int32_t)(((it.b * s.H + h) * s.M + it.c) * kN),
                                bar(B_HP_FULL));
                    ++n_hp;
                }
            }
        producer_end:
            for (int q = 0; q < kXSlots; ++q)
                if (last_x[q] >= 0)
                    mbar_drain(bar(B_X_FULL + q), (uint32_t)((last_x[q] / kXSlots) & 1));
            if (n_hp) mbar_drain(bar(B_HP_FULL), (n_hp - 1) & 1);
            if (n_items) mbar_drain(bar(B_ITEM_FULL), (n_items - 1) & 1);
        }
    } else if (warp == 1) {
        // -------------------------------- MMA ---------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kRows, 128, false, false);    // S = C B^T
            constexpr uint32_t idesc_h = idesc_bf16_f32(kRows, kP, false, true);      // C Hprev (bf16)
            constexpr uint32_t idesc_y = idesc_f32acc(kRows, kP, false, true, true);  // Y += P X (fp16)
            const uint64_t cdesc0 = smem_desc_sw128(sbase + kCOff, 16, 1024);
            uint32_t n_items = 0, n_hp = 0, n_x = 0, n_u = 0, n_y = 0;
            bool issued = false;
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const Item it = decode_item(p, k);
                if (item_rows(p, it) == 0) continue;
                const int nblk = (int)it.tau + 1;
                if (!mbar_wait(bar(B_ITEM_FULL), n_items & 1, abort_flag, err, 51)) goto mma_end;
                ++n_items;
                tc_fence_after();
                // units (head, block) in order; the P X product of a unit is issued one unit late, after the
                // next S, so that the tensor core works while builders make P. A head's accumulator is claimed
                // (and its Y_inter = C Hprev_h issued) just before the head's first P X, by which time the
                // epilogue has normally handed the previous head's accumulator back.
                int prev_sg = -1, prev_hh = -1;
                uint32_t prev_u = 0, prev_y = 0;
                for (int hh = 0; hh <= p.hpi; ++hh) {
                    for (int sg = 0; sg < nblk; ++sg) {
                        const bool real = hh < p.hpi;
                        if (real) {
                            if (sg == 0) ++n_y;  // a new head
                            // S = C B_sg^T into S buffer n_u % kSBufs, free once the P X of unit n_u - kSBufs is done
                            const int sb = (int)(n_u % kSBufs);
                            if (!mbar_wait(bar(B_S_EMPTY + sb), ((n_u / kSBufs) & 1) ^ 1, abort_flag, err, 54))
                                goto mma_end;
                            tc_fence_after();
                            const uint32_t ds = tmem + sb * 128;
                            const uint64_t bdesc0 = smem_desc_sw128(sbase + kBOff + sg * 2 * kBox, 16, 1024);
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint64_t off = (uint64_t)(((kk >> 2) * kBox + (kk & 3) * 32) >> 4);
                                mma_bf16(ds, cdesc0 + off, bdesc0 + off, idesc_s, kk > 0);
                            }
                            mma_commit(bar(B_S_FULL + sb));
                            issued = true;
                        }
                        if (prev_sg >= 0) {  // Y_intra += P X for the previous unit, P read from tensor memory
                            const int yb = (int)(prev_y % kYBufs);
                            if (prev_sg == 0) {  // the head's first P X: claim its accumulator, Y_inter = C Hprev_h
                                if (!mbar_wait(bar(B_Y_EMPTY + yb), ((prev_y / kYBufs) & 1) ^ 1, abort_flag, err, 52))
                                    goto mma_end;
                                if (!mbar_wait(bar(B_HP_FULL), n_hp & 1, abort_flag, err, 53)) goto mma_end;
                                tc_fence_after();
                                const uint32_t de = tmem + kYCol + yb * 128 + 64;
                                const uint64_t hdesc0 = smem_desc_sw128(sbase + kHpOff, 16384, 1024);
#pragma unroll
                                for (int kk = 0; kk < 8; ++kk)
                                    mma_bf16(de, cdesc0 + (uint64_t)(((kk >> 2) * kBox + (kk & 3) * 32) >> 4),
                                             hdesc0 + (uint64_t)((kk * 2048) >> 4), idesc_h, kk > 0);
                                mma_commit(bar(B_HP_EMPTY));
                                ++n_hp;
                                // the item's last C Hprev, after its last S: the C and B tiles are free and the
                                // next item's can load while the last P X products run
                                if (prev_hh == p.hpi - 1) mma_commit(bar(B_ITEM_EMPTY));
                            }
                            const int pb = (int)(prev_u % kSBufs);
                            // P_FULL also means the builders converted this unit's X slot (they waited for it)
                            if (!mbar_wait(bar(B_P_FULL + pb), (prev_u / kSBufs) & 1, abort_flag, err, 55)) goto mma_end;
                            const int xs = n_x % kXSlots;
                            tc_fence_after();
                            const uint32_t dy = tmem + kYCol + yb * 128;
                            const uint32_t pa = tmem + pb * 128;
                            const uint64_t xdesc0 = smem_desc_sw128(sbase + kXOff + xs * kBox, 16384, 1024);
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                // P of source tokens 0-63 sits in columns 0-31, of tokens 64-127 in 96-127
                                mma_f16_ts(dy, pa + (kk < 4 ? kk * 8 : 64 + kk * 8), xdesc0 + (uint64_t)((kk * 2048) >> 4),
                                           idesc_y, (prev_sg > 0 || kk > 0));
                            mma_commit(bar(B_S_EMPTY + pb));
                            mma_commit(bar(B_X_EMPTY + xs));
                            ++n_x;
                            if (prev_sg == nblk - 1) mma_commit(bar(B_Y_FULL + yb));
                        }
                        if (real) {
                            prev_sg = sg;
                            prev_hh = hh;
                            prev_u = n_u;
                            prev_y = n_y - 1;
                            ++n_u;
                        } else {
                            prev_sg = -1;
                            break;
                        }
                    }
                }
            }
        mma_end:
            if (issued) {
                mma_commit(bar(B_MMA_DONE));
                mbar_drain(bar(B_MMA_DONE), 0);
            }
        }
    } else if (warp < 10) {
        // ------------------------------ builders ------------------------------
        // two groups of four warps build every unit together: group g takes S columns 64g..64g+63 (the
        // unit's source tokens), so a unit's P is ready in half the time. A group writes its fp16 P over
        // S columns it has already read: group 0 into columns 0-31, group 1 into 96-127, working from its
        // upper 32-column block down.
        const int group = (warp - 2) >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int btid = (warp - 2) * 32 + lane;  // 0..255
        uint32_t n_u = 0, n_items = 0, n_sync = 0;
        // cs (log2 units) of an item's chunk for every head, this thread's token: fetched one item ahead, so
        // that the loads' latency falls inside the previous item's work
        auto next_live = [&](int64_t k2) {
            while (k2 < p.n_items && item_rows(p, decode_item(p, k2)) == 0) k2 = sched_next(k2);
            return k2;
        };
        auto fetch_cs = [&](int64_t k2, float (&v)[kHpi]) {
#pragma unroll
            for (int hh = 0; hh < kHpi; ++hh) v[hh] = 0.f;
            if (k2 >= p.n_items) return;
            const Item i2 = decode_item(p, k2);
            const int64_t clen2 = min(s.S, s.L - i2.c * s.S);
#pragma unroll
            for (int hh = 0; hh < kHpi; ++hh)
                if (hh < p.hpi && btid < clen2)
                    v[hh] = __ldg(p.cs + (i2.b * s.H + i2.hg * p.hpi + hh) * s.L + i2.c * s.S + btid) * kLog2e;
        };
        float cs_next[kHpi];
        fetch_cs(next_live(blockIdx.x), cs_next);
        for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
            const Item it = decode_item(p, k);
            if (item_rows(p, it) == 0) continue;
            const int nblk = (int)it.tau + 1;
            float *csi = cs_sm + (n_items & 1) * kHpi * 256;
            ++n_items;
#pragma unroll
            for (int hh = 0; hh < kHpi; ++hh) csi[hh * 256 + btid] = cs_next[hh];
            fetch_cs(next_live(sched_next(k)), cs_next);
            if (!group_sync(bar(B_GROUP), n_sync, abort_flag, err, 60)) goto builders_end;
            for (int hh = 0; hh < p.hpi; ++hh) {
                const float *csh = csi + hh * 256;
                const float cst = csh[it.tau * kRows + row];
                for (int sg = 0; sg < nblk; ++sg) {
                    const int sb = (int)(n_u % kSBufs);
                    if (!mbar_wait(bar(B_S_FULL + sb), (n_u / kSBufs) & 1, abort_flag, err, 61)) goto builders_end;
                    tc_fence_after();
                    const bool diag = sg == (int)it.tau;
                    const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + sb * 128;
                    // one 32-column block of S (q a compile-time constant)
                    auto block = [&](const int q) {
                        float v[32];
                        tmem_ld_32x32b_x32(ta + q * 32, v);
                        tmem_ld_wait();
                        uint32_t w[16];
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const float4 c4 = *reinterpret_cast<const float4 *>(csh + sg * kRows + q * 32 + 4 * j4);
                            const int c0 = q * 32 + 4 * j4;
                            float a0 = v[4 * j4] * ex2_approx(cst - c4.x);
                            float a1 = v[4 * j4 + 1] * ex2_approx(cst - c4.y);
                            float a2 = v[4 * j4 + 2] * ex2_approx(cst - c4.z);
                            float a3 = v[4 * j4 + 3] * ex2_approx(cst - c4.w);
                            if (diag) {
                                if (c0 > row) a0 = 0.f;
                                if (c0 + 1 > row) a1 = 0.f;
                                if (c0 + 2 > row) a2 = 0.f;
                                if (c0 + 3 > row) a3 = 0.f;
                            }
                            w[2 * j4] = pack_f16(a0, a1);
                            w[2 * j4 + 1] = pack_f16(a2, a3);
                        }
                        // P columns (two values per column) over S columns this group has already read
                        tmem_st_32x32b_x16(ta + (q < 2 ? q * 16 : 64 + q * 16), w);
                    };
#pragma unroll 1
                    for (int qi = 0; qi < 2; ++qi) block(group == 0 ? qi : 3 - qi);
                    tmem_st_wait();
                    {  // this unit's X block: bf16 -> fp16 in place, half by each group; consecutive lanes
                       // take consecutive 16-byte vectors, so a warp access touches 512 contiguous bytes
                        const int xs = n_u % kXSlots;
                        if (!mbar_wait(bar(B_X_FULL + xs), (n_u / kXSlots) & 1, abort_flag, err, 63)) goto builders_end;
                        uint4 *x4 = reinterpret_cast<uint4 *>(sm + kXOff + xs * kBox);
#pragma unroll
                        for (int q = 4 * group; q < 4 * group + 4; ++q) {
                            uint4 v = x4[row + 128 * q];
                            x4[row + 128 * q] = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y),
                                                           bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
                        }
                    }
                    fence_async_smem();  // the converted X is read by the tensor core (async proxy)
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(B_P_FULL + sb));
                    ++n_u;
                }
            }
        }
    builders_end:;
    } else {
        // ------------------------------ epilogue ------------------------------
        // Each warp owns two 4 KiB tiles (its 32 rows x one 32-column half of a head); Y goes through them
        // to the TMA store (per-lane accesses of 256-byte rows 8 KiB apart would split each warp
        // instruction into 32 line requests). Heads and halves are loops, not unrolled copies: the
        // kernel's warps run four different codes at once, and its speed follows the size of that code.
        const int quarter = warp & 3;  // the tensor-memory lane quarter this warp may read
        const int ew = warp - 10;      // this warp's tile pair
        const int row = quarter * 32 + lane;
        uint8_t *stg = sm + kStgOff + ew * 8192;
        uint32_t n_y = 0;
        // sum of y * 0 over every output: stays 0 unless a value is inf or NaN, which with finite inputs
        // means an fp16 operand (X, or P = (C_t . B_s) exp(cs_t - cs_s)) overflowed
        float nonfinite = 0.f;
        for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
            const Item it = decode_item(p, k);
            const int rows = item_rows(p, it);
            if (rows == 0) continue;
            const int64_t t = it.c * s.S + it.tau * kRows + row;
            const bool valid = row < rows;
            const int32_t ty = (int32_t)(it.c * s.S + it.tau * kRows + quarter * 32);  // first row of the warp
            const float *csrow = p.cs + (it.b * s.H + it.hg * p.hpi) * s.L + t;       // head hh at + hh * L
            float cs_next = valid ? __ldg(csrow) : 0.f;  // one head ahead, so the load overlaps the wait
#pragma unroll 1
            for (int hh = 0; hh < p.hpi; ++hh) {
                const int64_t h = it.hg * p.hpi + hh;
                const float decay = valid ? exp2f(cs_next * kLog2e) : 0.f;  // exp(cs_t)
                if (hh + 1 < p.hpi) cs_next = valid ? __ldg(csrow + (int64_t)(hh + 1) * s.L) : 0.f;
                const int yb = (int)(n_y % kYBufs);
                if (!mbar_wait(bar(B_Y_FULL + yb), (n_y / kYBufs) & 1, abort_flag, err, 71)) goto epilogue_end;
                tc_fence_after();
                __syncwarp();
                if (lane == 0) bulk_wait_group_read<0>();  // the tiles' last stores have read them
                __syncwarp();
                const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + kYCol + yb * 128;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float yi[32], ye[32];
                    tmem_ld_32x32b_x32(ta + half * 32, yi);
                    tmem_ld_32x32b_x32(ta + 64 + half * 32, ye);
                    tmem_ld_wait();
                    if (half == 1) {  // accumulators read: release them before the stores
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(B_Y_EMPTY + yb));
                    }
                    uint8_t *srow = stg + half * 4096 + lane * 128;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float4 *cell = reinterpret_cast<float4 *>(srow + ((q ^ (lane & 7)) << 4));
                        const float4 y = make_float4(fmaf(decay, ye[4 * q], yi[4 * q]),
                                                     fmaf(decay, ye[4 * q + 1], yi[4 * q + 1]),
                                                     fmaf(decay, ye[4 * q + 2], yi[4 * q + 2]),
                                                     fmaf(decay, ye[4 * q + 3], yi[4 * q + 3]));
                        nonfinite = fmaf(y.x, 0.f, fmaf(y.y, 0.f, fmaf(y.z, 0.f, fmaf(y.w, 0.f, nonfinite))));
                        *cell = y;
                    }
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {  // rows past the end of the batch row are clipped by the store
                        tma_store_3d(&tmY, smem_u32(stg + half * 4096), (int32_t)(h * kP + half * 32), ty,
                                     (int32_t)it.b);
                        bulk_commit_group();
                    }
                }
                ++n_y;
            }
        }
    epilogue_end:
        if (nonfinite != nonfinite && p.range) atomicOr(p.range, kRangeSsdOut);
        if (lane == 0) bulk_wait_group<0>();  // every store has landed before the CTA exits
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool ssd_tc_shape_ok(const Shape &s, bool bf16) {
    if (!bf16 || s.N != kN || s.P != kP || (s.S != 128 && s.S != 256)) return false;
    if (s.Bt * s.L >= (int64_t(1) << 31) || s.Bt * s.H * s.M * s.N >= (int64_t(1) << 31)) return false;
    return true;
}

cudaError_t launch_ssd_out_tc(const Shape &s, const LayerPtrs &lp, int *err_word, cudaStream_t st) {
    SsdTcParams p{};
    p.s = s;
    const int64_t hpg = s.H / s.G;
    p.hpi = hpg % kHpi == 0 ? kHpi : (hpg % 2 == 0 ? 2 : 1);
    p.ngh = (int)(s.H / p.hpi);
    p.ntiles = (int)(s.S / kRows);
    p.n_items = (int64_t)p.ntiles * s.Bt * s.M * p.ngh;
    p.cs = lp.cs;
    p.Y = static_cast<float *>(lp.Y);
    p.err = err_word;
    p.range = fp16_range_word();
    CUtensorMap mc, mb, mx, mh, my;
    const uint64_t gn = (uint64_t)(s.G * s.N);
    if (!make_tma_map_bf16(&mc, lp.C, gn, (uint64_t)(s.Bt * s.L), gn * 2, 64, 128) ||
        !make_tma_map_bf16(&mb, lp.B, gn, (uint64_t)(s.Bt * s.L), gn * 2, 64, 128) ||
        !make_tma_map_bf16(&mx, lp.X, (uint64_t)(s.H * s.P), (uint64_t)(s.Bt * s.L), (uint64_t)(s.H * s.P * 2), 64,
                           128) ||
        !make_tma_map_bf16(&mh, lp.Hprev, (uint64_t)s.P, (uint64_t)(s.Bt * s.H * s.M * s.N), (uint64_t)(s.P * 2), 64,
                           128) ||
        !make_tma_map_f32_3d(&my, lp.Y, (uint64_t)(s.H * s.P), (uint64_t)s.L, (uint64_t)s.Bt, (uint64_t)(s.H * s.P * 4),
                             (uint64_t)(s.L * s.H * s.P * 4), 32, 32))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k_ssd_out_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) {
        set_last_error("cudaFuncSetAttribute(ssd_out_tc)", e);
        return e;
    }
    const int64_t grid = std::min<int64_t>(p.n_items, device_sm_count());
    launch_begin(KK_SSD_OUT_TC, st);
    k_ssd_out_tc<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(mc, mb, mx, mh, my, p);
    return launch_end(KK_SSD_OUT_TC, st);
}

}  // namespace dart
