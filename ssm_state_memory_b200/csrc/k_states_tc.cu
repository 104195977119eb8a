// Chunk state memories on tcgen05 (DART paper §3 eq 5; App. A eq 20):
//
//   dH[b, h, c] = B_[c]^T diag(w_h) X_[c],h,   w_{s,h} = exp(Lambda_c - cs_s) = A_{s+1:e(c)}
//
// as one M=128 (n) x N=64*hpu (p of hpu heads) x K=S (tokens) GEMM per unit (batch, chunk, head pair).
// Units are taken in (b, c, head pair) order, heads fastest, and every CTA owns one contiguous range of
// them, so the chunk's B rows (shared by all heads of a group) are loaded and converted to fp16 once for
// up to H/2 units and a CTA changes chunks at most a few times. The X rows of a unit stream through a
// ring of 128-token stages; eight scaler warps give each thread one token row of one head, which it
// scales by w_s and converts to fp16 in place (the decay sits on the X side since B is shared across
// heads). fp16 keeps 11 mantissa bits for the scaled product (bf16 would keep 8). Two heads side by side
// form one N=128 MMA, halving the instruction count of N=64. The MMA writes fp32 into a 4-deep
// tensor-memory ring; four epilogue warps each write their 32 rows of dH as bf16 into a swizzled
// staging tile and hand it to a TMA store (per-thread 16-byte stores of 128-byte rows would spread every
// warp instruction over 32 lines and crowd the scalers out of the load/store pipe).
// Warps: 0 TMA producer, 1 MMA issuer, 2-9 scalers, 10-13 epilogue.
// Chunks shorter than a stage (S = 64, 32, 16): a unit is one 128-token span of a head pair (one head
// for S = 16), holding 128 / S chunks; each chunk's MMAs take only its own K rows (tokens) into an
// accumulator of its own, the scalers weight every row with the decay to the end of its own chunk, and
// the epilogue stores one chunk memory per accumulator.
// Needs chunk S in {16, 32, 64, 128, 256} and |B|, |w X| below the fp16 range limit (65504); beyond it
// the affected chunk memories are written as inf or NaN and the kernel raises kRangeChunkStates in the
// fp16 range word.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>

#include <algorithm>

#include "dart_internal.cuh"
#include "sm100_ptx.cuh"

namespace dart {
namespace {

using namespace sm100;

constexpr int kThreads = 448;
constexpr int kScalers = 8;                   // scaler warps 2..9
constexpr int kN = 128;
constexpr int kP = 64;
constexpr int kStages = 4;                    // X ring depth, 128 tokens x up to two heads per stage
constexpr int kDBufs = 4;
constexpr uint32_t kBox = 128 * 128;          // 128 rows x 128 bytes
constexpr uint32_t kBOff = 0;                 // B chunk: [s-block 0..1][n half 0..1] boxes
constexpr uint32_t kXOff = 4 * kBox;          // X ring: kStages stages of [head 0..1] boxes
constexpr uint32_t kStgOff = kXOff + kStages * 2 * kBox;  // dH staging: [epilogue warp][head] 32 x 128 B
constexpr uint32_t kBarOff = kStgOff + 4 * 2 * 4096;
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;
constexpr uint32_t kTmemCols = 512;           // kDBufs x 128 fp32 columns

enum {
    B_B_FULL = 0, B_B_EMPTY, B_B_READY, B_MMA_DONE, B_X_FULL, B_X_READY = B_X_FULL + kStages,
    B_X_EMPTY = B_X_READY + kStages, B_D_FULL = B_X_EMPTY + kStages, B_D_EMPTY = B_D_FULL + kDBufs,
    B_COUNT = B_D_EMPTY + kDBufs
};

struct StatesTcParams {
    Shape s;
    int hpu;             // heads per unit (2 when the heads of a group pair up, else 1)
    int nck;             // chunks per unit: 1 (S >= 128), or 128 / S for a 128-token span of short chunks
    int64_t nspan;       // units along a batch row: M, or ceil(L / 128) spans
    int64_t npu;         // units per (batch, chunk or span) = H / hpu
    int64_t n_units;
    const float *cs;     // [Bt, H, L]
    const float *lam;    // [Bt, H, M]
    __nv_bfloat16 *dH;   // [Bt, H, M, N, P]
    int *err;
    int *range;          // fp16 range flag word (kRangeChunkStates), or null
};

struct Unit {
    int64_t b, c, h0, key;  // key: the (batch, chunk, group) whose B rows the unit multiplies
};

__device__ __forceinline__ Unit decode_unit(const StatesTcParams &p, int64_t u) {
    Unit it;
    const int64_t hp = u % p.npu;
    const int64_t r = u / p.npu;
    it.c = r % p.nspan;  // the chunk, or the 128-token span of short chunks
    it.b = r / p.nspan;
    it.h0 = hp * p.hpu;
    it.key = r * p.s.G + it.h0 / (p.s.H / p.s.G);
    return it;
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, float scale) {
    return pack_f16(__uint_as_float(w << 16) * scale, __uint_as_float(w & 0xffff0000u) * scale);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Scales the 16-byte vectors [j0, j0 + NJ) of token row r of a 128-row swizzled box by sc, bf16 -> fp16
// in place. Lanes hold consecutive rows, so each quarter-warp touches eight distinct 16-byte bank
// groups (the 128-byte swizzle XORs the vector index with r mod 8).
template <int NJ>
__device__ __forceinline__ void scale_row(uint8_t *box, int r, int j0, float sc) {
    uint4 *q[NJ];
    uint4 v[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        q[j] = reinterpret_cast<uint4 *>(box + r * 128 + (((j0 + j) ^ (r & 7)) << 4));
        v[j] = *q[j];
    }
#pragma unroll
    for (int j = 0; j < NJ; ++j)
        *q[j] = make_uint4(bf16x2_to_f16x2(v[j].x, sc), bf16x2_to_f16x2(v[j].y, sc), bf16x2_to_f16x2(v[j].z, sc),
                           bf16x2_to_f16x2(v[j].w, sc));
}

__global__ void __launch_bounds__(kThreads, 1)
    k_chunk_states_tc(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmD, const StatesTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kBarOff);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kBarOff + B_COUNT * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kBarOff + B_COUNT * 8 + 4);
    auto bar = [&](int k) { return smem_u32(&bars[k]); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape &s = p.s;
    const int nck = p.nck;                       // chunks per unit
    const int64_t ulen = nck > 1 ? 128 : s.S;    // tokens per unit
    const int nsb = (int)(ulen / 128);           // 128-token stages per unit
    const int hpu = p.hpu;
    const int acols = 64 * hpu;                  // accumulator columns of one chunk
    const int dbufs = (int)(kTmemCols / (nck * acols)) > kDBufs ? kDBufs : (int)(kTmemCols / (nck * acols));
    int *err = p.err;
    // this CTA's contiguous range of units
    const int64_t u_begin = p.n_units * blockIdx.x / gridDim.x;
    const int64_t u_end = p.n_units * (blockIdx.x + 1) / gridDim.x;

    if (threadIdx.x == 0) {
        for (int k = 0; k < B_COUNT; ++k) {
            uint32_t cnt = 1;
            if (k == B_B_READY || (k >= B_X_READY && k < B_X_READY + kStages)) cnt = kScalers;
            if (k >= B_D_EMPTY && k < B_D_EMPTY + kDBufs) cnt = 4;
            mbar_init(bar(k), cnt);
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmD);
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
            uint32_t n_b = 0, n_st = 0;
            int64_t key = -1;
            int64_t last_st[kStages];
            for (int q = 0; q < kStages; ++q) last_st[q] = -1;
            for (int64_t u = u_begin; u < u_end; ++u) {
                const Unit it = decode_unit(p, u);
                const int64_t row0 = it.b * s.L + it.c * ulen;
                // the unit's X stages first: they only wait for ring slots, never for the B buffer
                for (int sb = 0; sb < nsb; ++sb) {
                    const int st = n_st % kStages;
                    if (!mbar_wait(bar(B_X_EMPTY + st), ((n_st / kStages) & 1) ^ 1, abort_flag, err, 81))
                        goto producer_end;
                    mbar_arrive_expect_tx(bar(B_X_FULL + st), hpu * kBox);
                    for (int hh = 0; hh < hpu; ++hh)
                        tma_load_2d(sbase + kXOff + (st * 2 + hh) * kBox, &tmX, (int32_t)((it.h0 + hh) * kP),
                                    (int32_t)(row0 + sb * 128), bar(B_X_FULL + st));
                    last_st[st] = n_st;
                    ++n_st;
                }
                if (it.key != key) {  // a new chunk (or group): reload B once the last MMA on the old one is done
                    key = it.key;
                    if (!mbar_wait(bar(B_B_EMPTY), (n_b & 1) ^ 1, abort_flag, err, 82)) goto producer_end;
                    mbar_arrive_expect_tx(bar(B_B_FULL), nsb * 2 * kBox);
                    const int64_t grp = it.key % s.G;
                    for (int sb = 0; sb < nsb; ++sb)
                        for (int kh = 0; kh < 2; ++kh)
                            tma_load_2d(sbase + kBOff + (sb * 2 + kh) * kBox, &tmB, (int32_t)(grp * kN + kh * 64),
                                        (int32_t)(row0 + sb * 128), bar(B_B_FULL));
                    ++n_b;
                }
            }
        producer_end:
            // no copy may still be writing shared memory when the CTA exits
            for (int q = 0; q < kStages; ++q)
                if (last_st[q] >= 0)
                    mbar_drain(bar(B_X_FULL + q), (uint32_t)((last_st[q] / kStages) & 1));
            if (n_b) mbar_drain(bar(B_B_FULL), (n_b - 1) & 1);
        }
    } else if (warp == 1) {
        // -------------------------------- MMA ---------------------------------
        if (lane == 0) {
            const uint32_t idesc = idesc_f32acc(kN, kP * hpu, true, true, true);  // A = B^T, B = wX (MN-major), fp16
            uint32_t n_b = 0, n_st = 0, n_u = 0;
            int64_t key = -1;
            bool issued = false;
            for (int64_t u = u_begin; u < u_end; ++u) {
                const Unit it = decode_unit(p, u);
                if (it.key != key) {
                    if (n_b > 0) mma_commit(bar(B_B_EMPTY));  // the old B is free once every MMA so far is done
                    key = it.key;
                    if (!mbar_wait(bar(B_B_READY), n_b & 1, abort_flag, err, 91)) goto mma_end;
                    ++n_b;
                }
                const int db = n_u % dbufs;
                if (!mbar_wait(bar(B_D_EMPTY + db), ((n_u / dbufs) & 1) ^ 1, abort_flag, err, 93)) goto mma_end;
                tc_fence_after();
                const uint32_t d = tmem + db * nck * acols;
                for (int sb = 0; sb < nsb; ++sb) {
                    const int st = n_st % kStages;
                    if (!mbar_wait(bar(B_X_READY + st), (n_st / kStages) & 1, abort_flag, err, 92)) goto mma_end;
                    tc_fence_after();
                    // A: the B rows of this stage, two 64-wide n blocks one box apart; B: the scaled X rows of
                    // the unit's heads, one box per head
                    const uint64_t adesc0 = smem_desc_sw128(sbase + kBOff + sb * 2 * kBox, kBox, 1024);
                    const uint64_t xdesc0 = smem_desc_sw128(sbase + kXOff + st * 2 * kBox, kBox, 1024);
                    if (nck == 1) {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t off = (uint64_t)((kk * 2048) >> 4);
                            mma_bf16(d, adesc0 + off, xdesc0 + off, idesc, (sb > 0 || kk > 0));
                        }
                    } else {
                        // chunk k of the span: its own K rows (16-token steps) into accumulator k
                        const int kpc = 8 / nck;
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t off = (uint64_t)((kk * 2048) >> 4);
                            mma_bf16(d + (kk / kpc) * acols, adesc0 + off, xdesc0 + off, idesc, kk % kpc != 0);
                        }
                    }
                    mma_commit(bar(B_X_EMPTY + st));
                    ++n_st;
                }
                mma_commit(bar(B_D_FULL + db));
                issued = true;
                ++n_u;
            }
        mma_end:
            if (issued) {
                mma_commit(bar(B_MMA_DONE));
                mbar_drain(bar(B_MMA_DONE), 0);
            }
        }
    } else if (warp < 2 + kScalers) {
        // ------------------------------- scalers ------------------------------
        // thread = one token row r of one 128-token stage; with two heads per unit the halves of the
        // group take one head each, with one head they split the row's eight vectors
        const int tid = threadIdx.x - 64;  // 0..255
        const int r = tid & 127;
        const int hsel = hpu == 2 ? (tid >> 7) : 0;
        const int j0 = hpu == 2 ? 0 : (tid >> 7) * 4;
        uint32_t n_b = 0, n_st = 0;
        int64_t key = -1;
        for (int64_t u = u_begin; u < u_end; ++u) {
            const Unit it = decode_unit(p, u);
            const int64_t clen = min(ulen, s.L - it.c * ulen);  // the unit's tokens
            const int64_t h = it.h0 + hsel;
            const float *csb = p.cs + (it.b * s.H + h) * s.L + it.c * ulen;
            for (int sb = 0; sb < nsb; ++sb) {
                const int st = n_st % kStages;
                const int srow = sb * 128 + r;
                // w_s = exp(Lambda of the row's chunk - cs_s), 0 past the end of the sequence
                const int64_t cch = nck > 1 ? it.c * nck + srow / s.S : it.c;
                const float sc = srow < clen ? expf(p.lam[(it.b * s.H + h) * s.M + cch] - csb[srow]) : 0.f;
                if (!mbar_wait(bar(B_X_FULL + st), (n_st / kStages) & 1, abort_flag, err, 101)) goto scalers_end;
                if (hpu == 2)
                    scale_row<8>(sm + kXOff + (st * 2 + hsel) * kBox, r, 0, sc);
                else
                    scale_row<4>(sm + kXOff + (st * 2 + hsel) * kBox, r, j0, sc);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_X_READY + st));
                ++n_st;
            }
            if (it.key != key) {
                key = it.key;
                if (!mbar_wait(bar(B_B_FULL), n_b & 1, abort_flag, err, 102)) goto scalers_end;
                ++n_b;
                // B rows bf16 -> fp16 in place; rows past the chunk end are zeroed
                for (int bx = tid >> 7; bx < nsb * 2; bx += 2) {
                    if ((bx >> 1) * 128 + r < clen) {
                        scale_row<8>(sm + kBOff + bx * kBox, r, 0, 1.f);
                    } else {
                        uint4 *row = reinterpret_cast<uint4 *>(sm + kBOff + bx * kBox + r * 128);
                        for (int j = 0; j < 8; ++j) row[j] = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_B_READY));
            }
        }
    scalers_end:;
    } else {
        // ------------------------------ epilogue ------------------------------
        const int quarter = warp & 3;  // the tensor-memory lane quarter this warp may read
        uint8_t *stg = sm + kStgOff + (warp - 2 - kScalers) * 2 * 4096;  // this warp's [head] 32 x 128 B tiles
        uint32_t n_u = 0;
        // sum of v * 0 over every value written: stays 0 unless a value is inf or NaN, which with finite
        // inputs means an fp16 operand (B, or a decay-scaled X) overflowed
        float nonfinite = 0.f;
        for (int64_t u = u_begin; u < u_end; ++u) {
            const Unit it = decode_unit(p, u);
            const int db = n_u % dbufs;
            if (!mbar_wait(bar(B_D_FULL + db), (n_u / dbufs) & 1, abort_flag, err, 111)) goto epilogue_end;
            tc_fence_after();
            for (int k = 0; k < nck; ++k) {  // the unit's chunks (one unless they are short)
                const int64_t chunk = it.c * nck + k;
                if (chunk >= s.M) break;  // a span past the last chunk of the row
                if (lane == 0) bulk_wait_group_read<0>();  // the previous stores have read the staging tiles
                __syncwarp();
                const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + (db * nck + k) * acols;
                for (int hh = 0; hh < hpu; ++hh) {
                    // state row quarter*32 + lane; its 64 p values go to staging row `lane`, 128-byte swizzled
                    uint8_t *row = stg + hh * 4096 + lane * 128;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float v[32];
                        tmem_ld_32x32b_x32(ta + hh * 64 + half * 32, v);
                        tmem_ld_wait_32(v);
#pragma unroll
                        for (int q = 0; q < 32; ++q) nonfinite = fmaf(v[q], 0.f, nonfinite);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<uint4 *>(row + (((half * 4 + q) ^ (lane & 7)) << 4)) =
                                make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                                           pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    for (int hh = 0; hh < hpu; ++hh)
                        tma_store_2d(&tmD, smem_u32(stg + hh * 4096), 0,
                                     (int32_t)(((it.b * s.H + it.h0 + hh) * s.M + chunk) * kN + quarter * 32));
                    bulk_commit_group();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_D_EMPTY + db));
            ++n_u;
        }
    epilogue_end:
        if (nonfinite != nonfinite && p.range) atomicOr(p.range, kRangeChunkStates);
        if (lane == 0) bulk_wait_group<0>();  // every dH store has landed before the CTA exits
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool states_tc_shape_ok(const Shape &s, bool bf16) {
    if (!bf16 || s.N != kN || s.P != kP || (s.S != 16 && s.S != 32 && s.S != 64 && s.S != 128 && s.S != 256))
        return false;
    if (s.Bt * s.L >= (int64_t(1) << 31)) return false;
    if (s.Bt * s.H * s.M * kN >= (int64_t(1) << 31)) return false;  // dH rows addressed by the TMA store
    return true;
}

cudaError_t launch_chunk_states_tc(const Shape &s, const LayerPtrs &lp, int *err_word, cudaStream_t st) {
    StatesTcParams p{};
    p.s = s;
    p.nck = s.S >= 128 ? 1 : (int)(128 / s.S);
    // two heads a unit when the heads of a group pair up, except with 8 chunks a unit (S = 16): their
    // 8 accumulators of 128 columns would not fit the 512 of tensor memory, 8 of 64 do
    p.hpu = ((s.H / s.G) % 2 == 0 && p.nck < 8) ? 2 : 1;
    p.npu = s.H / p.hpu;
    p.nspan = s.S >= 128 ? s.M : (s.L + 127) / 128;
    p.n_units = s.Bt * p.nspan * p.npu;
    p.cs = lp.cs;
    p.lam = lp.lam;
    p.dH = static_cast<__nv_bfloat16 *>(lp.dH);
    p.err = err_word;
    p.range = fp16_range_word();
    CUtensorMap mb, mx, md;
    const uint64_t gn = (uint64_t)(s.G * s.N);
    if (!make_tma_map_bf16(&mb, lp.B, gn, (uint64_t)(s.Bt * s.L), gn * 2, 64, 128) ||
        !make_tma_map_bf16(&mx, lp.X, (uint64_t)(s.H * s.P), (uint64_t)(s.Bt * s.L), (uint64_t)(s.H * s.P * 2), 64,
                           128) ||
        !make_tma_map_bf16(&md, lp.dH, (uint64_t)kP, (uint64_t)(s.Bt * s.H * s.M * kN), (uint64_t)(kP * 2), 64, 32))
        return cudaErrorInvalidValue;
    cudaError_t e =
        cudaFuncSetAttribute(k_chunk_states_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) {
        set_last_error("cudaFuncSetAttribute(chunk_states_tc)", e);
        return e;
    }
    const int64_t grid = std::min<int64_t>(p.n_units, device_sm_count());
    launch_begin(KK_CHUNK_STATES_TC, st);
    k_chunk_states_tc<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(mb, mx, md, p);
    return launch_end(KK_CHUNK_STATES_TC, st);
}

}  // namespace dart
