// Chunk state memories on tcgen05 (DART paper §3 eq 5; App. A eq 20):
//
//   dH[b, h, c] = B_[c]^T diag(w_h) X_[c],h,   w_{s,h} = exp(Lambda_c - cs_s) = A_{s+1:e(c)}
//
// as one M=128 (n) x N=64 (p) x K=S (tokens) GEMM per (batch, chunk, head).
// Work item = (chunk c, batch b, 4 heads). The chunk's B rows (shared by all
// heads, G = 1) are loaded once per item and converted to fp16 in place; per head
// the X block streams through a 4-slot ring, where four warps scale each token row
// by w_s and convert it to fp16 in place (the decay must sit on the X side, since
// B is shared across heads and w is per head). fp16 keeps 11 mantissa bits for the
// scaled product (bf16 would keep 8). The MMA writes fp32 into a 4-deep
// tensor-memory ring and four epilogue warps store bf16 rows of dH.
// Warps: 0 TMA producer, 1 MMA issuer, 2-5 scalers, 6-9 epilogue.
// Needs chunk S in {128, 256} and |B|, |w X| below the fp16 range limit (65504).
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>

#include <algorithm>

#include "dart_internal.cuh"
#include "sm100_ptx.cuh"

namespace dart {
namespace {

using namespace sm100;

constexpr int kThreads = 320;
constexpr int kN = 128;
constexpr int kP = 64;
constexpr int kHpi = 4;
constexpr int kXSlots = 4;
constexpr int kDBufs = 4;
constexpr uint32_t kBox = 128 * 128;          // 128 rows x 128 bytes
constexpr uint32_t kBOff = 0;                 // B chunk: [s-block 0..1][n half 0..1] boxes
constexpr uint32_t kXOff = 4 * kBox;          // X ring: kXSlots slots of [s-block 0..1] boxes
constexpr uint32_t kWOff = kXOff + kXSlots * 2 * kBox;  // decay weights w[head][token] of the item (fp32)
constexpr uint32_t kBarOff = kWOff + kHpi * 256 * 4;
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;
constexpr uint32_t kTmemCols = 256;

enum {
    B_ITEM_FULL = 0, B_ITEM_EMPTY, B_B_READY, B_MMA_DONE, B_X_FULL, B_X_READY = B_X_FULL + kXSlots,
    B_X_EMPTY = B_X_READY + kXSlots, B_D_FULL = B_X_EMPTY + kXSlots, B_D_EMPTY = B_D_FULL + kDBufs,
    B_GROUP = B_D_EMPTY + kDBufs, B_COUNT
};

struct StatesTcParams {
    Shape s;
    int hpi, ngh;
    int64_t n_items;
    const float *cs;    // [Bt, H, L]
    const float *lam;   // [Bt, H, M]
    __nv_bfloat16 *dH;  // [Bt, H, M, N, P]
    int *err;
};

struct Item {
    int64_t b, c, hg;
};

__device__ __forceinline__ Item decode_item(const StatesTcParams &p, int64_t k) {
    Item it;
    it.c = k / (p.s.Bt * p.ngh);
    int64_t r = k % (p.s.Bt * p.ngh);
    it.b = r / p.ngh;
    it.hg = r % p.ngh;
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

__global__ void __launch_bounds__(kThreads, 1)
    k_chunk_states_tc(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmX,
                      const StatesTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kBarOff);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kBarOff + B_COUNT * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kBarOff + B_COUNT * 8 + 4);
    auto bar = [&](int k) { return smem_u32(&bars[k]); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape &s = p.s;
    const int nsb = (int)(s.S / 128);  // 128-token blocks per chunk
    int *err = p.err;

    if (threadIdx.x == 0) {
        for (int k = 0; k < B_COUNT; ++k) {
            uint32_t cnt = 1;
            // one arrival per scaler / epilogue warp (B_D_EMPTY..: epilogue; B_GROUP: scalers)
            if (k == B_B_READY || (k >= B_X_READY && k < B_X_READY + kXSlots) || (k >= B_D_EMPTY && k < B_COUNT))
                cnt = 4;
            mbar_init(bar(k), cnt);
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmX);
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
            uint32_t n_items = 0, n_x = 0;
            int64_t last_x[kXSlots];
            for (int q = 0; q < kXSlots; ++q) last_x[q] = -1;
            for (int64_t k = blockIdx.x; k < p.n_items; k += gridDim.x) {
                const Item it = decode_item(p, k);
                const int64_t h0 = it.hg * p.hpi;
                const int64_t grp = h0 / (s.H / s.G);
                if (!mbar_wait(bar(B_ITEM_EMPTY), (n_items & 1) ^ 1, abort_flag, err, 81)) goto producer_end;
                mbar_arrive_expect_tx(bar(B_ITEM_FULL), nsb * 2 * kBox);
                for (int sb = 0; sb < nsb; ++sb)
                    for (int kh = 0; kh < 2; ++kh)
                        tma_load_2d(sbase + kBOff + (sb * 2 + kh) * kBox, &tmB, (int32_t)(grp * kN + kh * 64),
                                    (int32_t)(it.b * s.L + it.c * s.S + sb * 128), bar(B_ITEM_FULL));
                ++n_items;
                for (int hh = 0; hh < p.hpi; ++hh) {
                    const int64_t h = h0 + hh;
                    const int slot = n_x % kXSlots;
                    if (!mbar_wait(bar(B_X_EMPTY + slot), ((n_x / kXSlots) & 1) ^ 1, abort_flag, err, 82))
                        goto producer_end;
                    mbar_arrive_expect_tx(bar(B_X_FULL + slot), nsb * kBox);
                    for (int sb = 0; sb < nsb; ++sb)
                        tma_load_2d(sbase + kXOff + (slot * 2 + sb) * kBox, &tmX, (int32_t)(h * kP),
                                    (int32_t)(it.b * s.L + it.c * s.S + sb * 128), bar(B_X_FULL + slot));
                    last_x[slot] = n_x;
                    ++n_x;
                }
            }
        producer_end:
            for (int q = 0; q < kXSlots; ++q)
                if (last_x[q] >= 0)
                    mbar_wait(bar(B_X_FULL + q), (uint32_t)((last_x[q] / kXSlots) & 1), abort_flag, nullptr, 0);
            if (n_items) mbar_wait(bar(B_ITEM_FULL), (n_items - 1) & 1, abort_flag, nullptr, 0);
        }
    } else if (warp == 1) {
        // -------------------------------- MMA ---------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f32acc(kN, kP, true, true, true);  // A = B^T (MN-major), fp16
            uint32_t n_items = 0, n_x = 0;
            bool issued = false;
            for (int64_t k = blockIdx.x; k < p.n_items; k += gridDim.x) {
                if (!mbar_wait(bar(B_B_READY), n_items & 1, abort_flag, err, 91)) goto mma_end;
                ++n_items;
                for (int hh = 0; hh < p.hpi; ++hh) {
                    const int slot = n_x % kXSlots;
                    const int db = n_x % kDBufs;
                    if (!mbar_wait(bar(B_X_READY + slot), (n_x / kXSlots) & 1, abort_flag, err, 92)) goto mma_end;
                    if (!mbar_wait(bar(B_D_EMPTY + db), ((n_x / kDBufs) & 1) ^ 1, abort_flag, err, 93)) goto mma_end;
                    tc_fence_after();
                    const uint32_t d = tmem + db * kP;
                    for (int sb = 0; sb < nsb; ++sb) {
                        // A: the B rows of this block, two 64-wide n blocks 16 KiB apart; B: the scaled X rows
                        const uint64_t adesc0 = smem_desc_sw128(sbase + kBOff + sb * 2 * kBox, kBox, 1024);
                        const uint64_t xdesc0 = smem_desc_sw128(sbase + kXOff + (slot * 2 + sb) * kBox, kBox, 1024);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t off = (uint64_t)((kk * 2048) >> 4);
                            mma_bf16(d, adesc0 + off, xdesc0 + off, idesc, (sb > 0 || kk > 0));
                        }
                    }
                    mma_commit(bar(B_X_EMPTY + slot));
                    mma_commit(bar(B_D_FULL + db));
                    issued = true;
                    ++n_x;
                }
                mma_commit(bar(B_ITEM_EMPTY));
            }
        mma_end:
            if (issued) {
                mma_commit(bar(B_MMA_DONE));
                mbar_wait(bar(B_MMA_DONE), 0, abort_flag, nullptr, 0);
            }
        }
    } else if (warp < 6) {
        // ------------------------------- scalers ------------------------------
        const int tid = threadIdx.x - 64;  // 0..127
        float *wsm = reinterpret_cast<float *>(sm + kWOff);
        uint32_t n_items = 0, n_x = 0, n_sync = 0;
        for (int64_t k = blockIdx.x; k < p.n_items; k += gridDim.x) {
            const Item it = decode_item(p, k);
            const int64_t clen = min(s.S, s.L - it.c * s.S);
            // decay weights of every head of the item, w = exp(Lambda_c - cs_s) (0 past the chunk end);
            // the previous item's conversions are finished, so the array is free
            for (int hh = 0; hh < p.hpi; ++hh) {
                const int64_t h = it.hg * p.hpi + hh;
                const float total = p.lam[(it.b * s.H + h) * s.M + it.c];
                const float *csb = p.cs + (it.b * s.H + h) * s.L + it.c * s.S;
                for (int srow = tid; srow < 256; srow += 128)
                    wsm[hh * 256 + srow] = srow < clen ? expf(total - csb[srow]) : 0.f;
            }
            if (!group_sync(bar(B_GROUP), n_sync, abort_flag, err, 100)) goto scalers_end;
            if (!mbar_wait(bar(B_ITEM_FULL), n_items & 1, abort_flag, err, 101)) goto scalers_end;
            ++n_items;
            {  // B chunk bf16 -> fp16 in place (rows past the chunk end are zeroed); lane-contiguous vectors
                uint4 *b4 = reinterpret_cast<uint4 *>(sm + kBOff);
                for (int i = tid; i < nsb * 2 * (int)kBox / 16; i += 128) {
                    const int srow = (i / 8) % 128 + ((i / 8) / 256) * 128;  // box = (s-block, n half), 8 vectors/row
                    uint4 v = b4[i];
                    b4[i] = srow < clen ? make_uint4(bf16x2_to_f16x2(v.x, 1.f), bf16x2_to_f16x2(v.y, 1.f),
                                                     bf16x2_to_f16x2(v.z, 1.f), bf16x2_to_f16x2(v.w, 1.f))
                                        : make_uint4(0u, 0u, 0u, 0u);
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_B_READY));
            for (int hh = 0; hh < p.hpi; ++hh) {
                const int slot = n_x % kXSlots;
                if (!mbar_wait(bar(B_X_FULL + slot), (n_x / kXSlots) & 1, abort_flag, err, 102)) goto scalers_end;
                // X rows scaled by w and converted to fp16 in place; vector i of the slot is token row
                // (i / 8) of its 128-row box, lanes take consecutive vectors (conflict-free)
                uint4 *x4 = reinterpret_cast<uint4 *>(sm + kXOff + slot * 2 * kBox);
                for (int i = tid; i < nsb * (int)kBox / 16; i += 128) {
                    const float sc = wsm[hh * 256 + (i >> 3)];
                    uint4 v = x4[i];
                    x4[i] = make_uint4(bf16x2_to_f16x2(v.x, sc), bf16x2_to_f16x2(v.y, sc), bf16x2_to_f16x2(v.z, sc),
                                       bf16x2_to_f16x2(v.w, sc));
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_X_READY + slot));
                ++n_x;
            }
            // all conversions of this item read wsm before it is rewritten
            if (!group_sync(bar(B_GROUP), n_sync, abort_flag, err, 103)) goto scalers_end;
        }
    scalers_end:;
    } else {
        // ------------------------------ epilogue ------------------------------
        const int quarter = warp & 3;
        const int n = quarter * 32 + lane;  // state row
        uint32_t n_x = 0;
        for (int64_t k = blockIdx.x; k < p.n_items; k += gridDim.x) {
            const Item it = decode_item(p, k);
            for (int hh = 0; hh < p.hpi; ++hh) {
                const int64_t h = it.hg * p.hpi + hh;
                const int db = n_x % kDBufs;
                if (!mbar_wait(bar(B_D_FULL + db), (n_x / kDBufs) & 1, abort_flag, err, 111)) goto epilogue_end;
                tc_fence_after();
                const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + db * kP;
                uint4 *dst = reinterpret_cast<uint4 *>(p.dH + (((it.b * s.H + h) * s.M + it.c) * kN + n) * kP);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float v[32];
                    tmem_ld_32x32b_x32(ta + half * 32, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[half * 4 + q] = make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                                                       pack_bf16(v[8 * q + 4], v[8 * q + 5]),
                                                       pack_bf16(v[8 * q + 6], v[8 * q + 7]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_D_EMPTY + db));
                ++n_x;
            }
        }
    epilogue_end:;
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
    if (!bf16 || s.N != kN || s.P != kP || (s.S != 128 && s.S != 256)) return false;
    if (s.Bt * s.L >= (int64_t(1) << 31)) return false;
    return true;
}

cudaError_t launch_chunk_states_tc(const Shape &s, const LayerPtrs &lp, int *err_word, cudaStream_t st) {
    StatesTcParams p{};
    p.s = s;
    const int64_t hpg = s.H / s.G;
    p.hpi = hpg % kHpi == 0 ? kHpi : (hpg % 2 == 0 ? 2 : 1);
    p.ngh = (int)(s.H / p.hpi);
    p.n_items = s.M * s.Bt * p.ngh;
    p.cs = lp.cs;
    p.lam = lp.lam;
    p.dH = static_cast<__nv_bfloat16 *>(lp.dH);
    p.err = err_word;
    CUtensorMap mb, mx;
    const uint64_t gn = (uint64_t)(s.G * s.N);
    if (!make_tma_map_bf16(&mb, lp.B, gn, (uint64_t)(s.Bt * s.L), gn * 2, 64, 128) ||
        !make_tma_map_bf16(&mx, lp.X, (uint64_t)(s.H * s.P), (uint64_t)(s.Bt * s.L), (uint64_t)(s.H * s.P * 2), 64,
                           128))
        return cudaErrorInvalidValue;
    cudaError_t e =
        cudaFuncSetAttribute(k_chunk_states_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) {
        set_last_error("cudaFuncSetAttribute(chunk_states_tc)", e);
        return e;
    }
    const int64_t grid = std::min<int64_t>(p.n_items, device_sm_count());
    launch_begin(KK_CHUNK_STATES_TC, st);
    k_chunk_states_tc<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(mb, mx, p);
    return launch_end(KK_CHUNK_STATES_TC, st);
}

}  // namespace dart
