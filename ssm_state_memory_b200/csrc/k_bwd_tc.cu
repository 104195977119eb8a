// tcgen05 kernels of the SMA backward (bf16, N = 128, P = 64, S a multiple of 128 or a divisor of 128).
//
// The backward of state-memory attention (DART §3 eq 8-10) by recomputation (§4
// "Efficient Training"; App. C eq 32-35): the forward kept only R and lse. Per token t,
// head h and historical chunk c < chunk(t):
//   U = Q_t dH[c], V = C_t dH[c] (P-vectors), l = U . E_t / sqrt(N), w = exp(l - lse_t),
//   dw = dR_t . V, D_t = dR_t . R_t, a = w (dw - D_t) / sqrt(N),
//   dE_t += a U,   dQ_t += a dH[c] E_t,   dC_t += w dH[c] dR_t,
//   ddH[c] += Q_t^T (a E_t) + C_t^T (w dR_t).
//
// Launches:
//   prep      D_t = dR_t . R_t (fp32).
//   recompute (k_sma_bwd_r_tc) one item = a 128-token tile of one chunk and a group of heads,
//             as in the forward. Per head pair and historical chunk j the tensor cores form
//             U = Q [dH_h | dH_h+1] and V = C [dH_h | dH_h+1] into one of two tensor-memory
//             buffers; the warp that owns a token row forms w, dw (fp32 dR), a, accumulates
//             dE += a U in registers, and writes the pair's scalars a and w to the workspace
//             (2 floats per token, chunk and head): the chunk weights of the recomputation.
//   gradient GEMMs (k_sma_bwd_gq_tc, k_sma_bwd_gm_tc) contract the scalar-weighted rows
//             a E_t and w dR_t with the chunk memories (dQ, dC: K = P) and with Q and C (ddH:
//             K = the tokens of a tile), all operands in fp16 (11 significant bits): dH, Q and
//             C as fp16 copies (k_bwd_to_f16; exact for bf16 values in fp16 range), the rows
//             rounded once after a power-of-two scale that puts the largest row value of the
//             whole backward between 2^13 and 2^14 (the recompute kernel and the D pass find
//             the maxima of |a E_t| and |dR|); the accumulators are scaled back in fp32. A
//             single bf16 rounding of the rows (8 bits) moved the heavy-tailed dQ (max/rms near
//             40) by 2.3e-2 of its rms; fp16 moves it by about 5e-3.
// Tokens of chunk 0 get zero dQ, dC, dE (written by the host before the launches).
#include <cuda.h>
#include <math.h>

#include <algorithm>
#include <cstdio>

#include <cuda_fp16.h>

#include "dart_internal.cuh"
#include "sm100_ptx.cuh"

namespace dart {

namespace {

using namespace sm100;

constexpr int kN = 128, kP = 64, kTile = 128;
constexpr uint32_t kBox = 128 * 128;  // one 128-row x 128-byte TMA box
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRs = 0.08838834764831845f;  // 1 / sqrt(N), N = 128

__device__ __forceinline__ void fence_async_smem_b() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void lds128(uint32_t a, uint32_t &x, uint32_t &y, uint32_t &z, uint32_t &w) {
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(x), "=r"(y), "=r"(z), "=r"(w) : "r"(a) : "memory");
}

__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// x = hi + lo with hi = bf16(x) and lo = bf16(x - hi), for two values at once (bf16 pairs):
// hi + lo carries 16 significant bits of x
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - __low2float(h), x1 - __high2float(h));
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// 2^(14 - e) for the largest magnitude m (the bits of a non-negative float) with m < 2^e, so that every
// value up to m scales to below 2^14; 1 when m is 0 or not finite
__device__ __forceinline__ float pow2_scale(unsigned bits) {
    const int ex = (int)((bits >> 23) & 0xffu);
    if (bits == 0u || ex == 0xff) return 1.f;
    const int sh = max(-100, min(100, 14 - (ex - 126)));
    return __int_as_float((127 + sh) << 23);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

struct QItem {
    int64_t i, b, tile, hg;
};

// item k of the query-tile kernels: (slot i descending, batch row, tile of the slot, head group). With
// S a multiple of 128 a slot is a chunk and its tiles are the chunk's 128-token tiles; with S < 128
// (S dividing 128) a slot is one 128-token tile, which spans 128 / S chunks (multi).
__device__ __forceinline__ QItem q_item(const Shape &s, int ntiles, int ngh, int64_t nslot, int64_t k) {
    const uint32_t per_b = (uint32_t)ntiles * (uint32_t)ngh, per_i = (uint32_t)s.Bt * per_b;
    const uint32_t k32 = (uint32_t)k;
    QItem it;
    const uint32_t q = k32 / per_i;
    it.i = nslot - 1 - (int64_t)q;
    uint32_t r = k32 - q * per_i;
    const uint32_t b = r / per_b;
    r -= b * per_b;
    const uint32_t tile = r / (uint32_t)ngh;
    it.b = b;
    it.tile = tile;
    it.hg = r - tile * (uint32_t)ngh;
    return it;
}

// first token of the item's tile
__device__ __forceinline__ int64_t q_t0(const Shape &s, const QItem &it, bool multi) {
    return multi ? it.i * kTile : it.i * s.S + it.tile * kTile;
}

__device__ __forceinline__ int q_rows(const Shape &s, const QItem &it, bool multi) {
    const int64_t t0 = q_t0(s, it, multi);
    const int64_t end = multi ? s.L : min(s.L, (it.i + 1) * s.S);
    return (int)max((int64_t)0, min((int64_t)kTile, end - t0));
}

// chunk steps of the item: the chunks before its last row's chunk (every row of a one-chunk tile has
// chunk i; in a multi-chunk tile each row takes only the steps below its own chunk)
__device__ __forceinline__ int64_t q_steps(const Shape &s, const QItem &it, bool multi, int rows) {
    if (rows <= 0) return 0;
    return multi ? (q_t0(s, it, true) + rows - 1) / s.S : it.i;
}

// ---------------------------------------------------------------------------
// prep: D[b, h, t] = dR_t . R_t over the (b, t, h) rows of 64 floats. A half-warp takes a row (16-byte
// loads), a warp four rows per pass (two per half), all eight loads issued before the first product, so
// that enough bytes are in flight to stream R and dR at HBM speed.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_sma_bwd_prep(Shape s, const float *__restrict__ R,
                                                       const float *__restrict__ dR, float *__restrict__ D,
                                                       unsigned *dr_max) {
    const int lane = threadIdx.x & 31, hl = lane & 15, half = lane >> 4;
    const int64_t rows = s.Bt * s.L * s.H;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    float mx = 0.f;  // of |dR| over this lane's loads
    for (int64_t r0 = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * 4; r0 < rows; r0 += nw * 4) {
        float4 g[2], a[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t r = r0 + 2 * u + half;
            if (r < rows) {
                g[u] = __ldg(reinterpret_cast<const float4 *>(dR + r * kP) + hl);
                a[u] = __ldg(reinterpret_cast<const float4 *>(R + r * kP) + hl);
            } else {
                g[u] = a[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(g[u].x), fabsf(g[u].y)), fmaxf(fabsf(g[u].z), fabsf(g[u].w))));
            float acc = fmaf(g[u].x, a[u].x, fmaf(g[u].y, a[u].y, fmaf(g[u].z, a[u].z, g[u].w * a[u].w)));
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            const int64_t r = r0 + 2 * u + half;
            if (hl == 0 && r < rows) {
                const int64_t h = r % s.H, bt = r / s.H;
                D[(bt / s.L * s.H + h) * s.L + bt % s.L] = acc;
            }
        }
    }
    mx = warp_max(mx);
    if (dr_max && lane == 0) atomicMax(dr_max, __float_as_uint(mx));
}

// ---------------------------------------------------------------------------
// fp16 copies of dH, Q and C for the gradient GEMMs: exact for bf16 values from 2^-17 up to 65280; a
// value of 65536 or more (or inf, NaN) becomes inf or NaN there and raises kRangeBwdOperands.
// ---------------------------------------------------------------------------
struct F16Copy {
    const uint4 *src;
    uint4 *dst;
    int64_t n;  // 16-byte vectors (8 values)
};

__global__ void __launch_bounds__(256) k_bwd_to_f16(const F16Copy c0, const F16Copy c1, const F16Copy c2,
                                                     int *range) {
    const int64_t n01 = c0.n + c1.n, ntot = n01 + c2.n;
    bool over = false;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < ntot; i += (int64_t)gridDim.x * blockDim.x) {
        const bool in0 = i < c0.n, in1 = !in0 && i < n01;
        const uint4 *src = in0 ? c0.src : (in1 ? c1.src : c2.src);
        uint4 *dst = in0 ? c0.dst : (in1 ? c1.dst : c2.dst);
        const int64_t j = in0 ? i : (in1 ? i - c0.n : i - n01);
        const uint4 v = __ldg(src + j);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            over |= (w[k] & 0x7fffu) >= 0x4780u || (w[k] & 0x7fff0000u) >= 0x47800000u;
            o[k] = pack_f16x2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xffff0000u));
        }
        dst[j] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (__any_sync(0xffffffffu, over) && (threadIdx.x & 31) == 0 && range) atomicOr(range, kRangeBwdOperands);
}

// ---------------------------------------------------------------------------
// recompute: dE (tensor memory), and the scalars a, w of every (token, chunk, head)
// ---------------------------------------------------------------------------
constexpr int kRThreads = 384;  // warp 0 TMA, warp 1 MMA, warps 2-3 idle, warps 4-11 per-token work
constexpr int kRRegsLaunch = 168, kRRegsLow = 80, kRRegsHigh = 208;
static_assert(128 * kRRegsLow + 256 * kRRegsHigh <= kRThreads * kRRegsLaunch, "register split exceeds the pool");
constexpr int kRStages = 2;                  // dH ring (a stage = a head pair's chunk memories)
constexpr uint32_t kR_Q = 0;                 // Q tile, two 64-column boxes
constexpr uint32_t kR_C = 2 * kBox;          // C tile
constexpr uint32_t kR_H = 4 * kBox;          // dH stages [stage][head of pair]
constexpr uint32_t kR_STG = kR_H + kRStages * 2 * kBox;  // per warp 12 KiB: E, dR hi, dR lo rows (32 x 128 B)
constexpr uint32_t kR_BAR = kR_STG + 8 * 12288;
constexpr uint32_t kR_SMEM = kR_BAR + 256 + 1024;
static_assert(kR_SMEM <= 232448, "recompute kernel exceeds the shared memory of a CTA");
constexpr uint32_t kRT_U = 0, kRT_V = 128;  // tensor-memory columns within each of the two 256-column buffers

enum { RB_QC_FULL = 0, RB_QC_EMPTY, RB_MMA_DONE, RB_MMA_DONE2, RB_ST_FULL, RB_ST_EMPTY = RB_ST_FULL + kRStages,
       RB_UV_FULL = RB_ST_EMPTY + kRStages, RB_UV_EMPTY = RB_UV_FULL + 2, RB_LD = RB_UV_EMPTY + 2,
       RB_COUNT = RB_LD + 8 };
static_assert(RB_COUNT * 8 + 8 <= 256, "barrier block overflows its 256 bytes");

struct BwdRParams {
    Shape s;
    int hpi, ngh, ntiles, multi;  // multi: 128-token tiles spanning several chunks (S < 128)
    int64_t nslot, n_items;
    const float *lse, *D;
    float *Wsc, *Asc;  // [Bt, H, M, L]: w and a of every (token, chunk, head)
    unsigned *amax;    // a bound on |a E_t,p| over every (token, chunk, head, p), as float bits (or null)
    int e_hpg;         // heads per E group (E and dE rows of head h are group h / e_hpg); 0 or 1: E per head
};

__global__ void __launch_bounds__(kRThreads, 1)
    k_sma_bwd_r_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC,
                   const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmE,
                   const __grid_constant__ CUtensorMap tmDR, const __grid_constant__ CUtensorMap tmDE,
                   const BwdRParams p, int *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kR_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kR_BAR + RB_COUNT * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kR_BAR + RB_COUNT * 8 + 4);
    auto bar = [&](int k) { return smem_u32(&bars[k]); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape &s = p.s;
    if (threadIdx.x == 0) {
        mbar_init(bar(RB_QC_FULL), 1);
        mbar_init(bar(RB_QC_EMPTY), 2);  // both MMA issuers commit when their MMAs of an item are done
        mbar_init(bar(RB_MMA_DONE), 1);
        mbar_init(bar(RB_MMA_DONE2), 1);
        for (int q = 0; q < kRStages; ++q) {
            mbar_init(bar(RB_ST_FULL + q), 1);
            mbar_init(bar(RB_ST_EMPTY + q), 1);
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(bar(RB_UV_FULL + q), 1);
            mbar_init(bar(RB_UV_EMPTY + q), 8);  // every per-token warp has read U and V
        }
        for (int w = 0; w < 8; ++w) mbar_init(bar(RB_LD + w), 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmH);
        tma_prefetch_desc(&tmE);
        tma_prefetch_desc(&tmDR);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        setmaxnreg_dec<kRRegsLow>();
        if (lane == 0) {
            uint32_t qc_uses = 0, ph = 0;
            int st = 0;
            int last_ph[kRStages];
            for (int q = 0; q < kRStages; ++q) last_ph[q] = -1;
            bool qc_loaded = false;
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const QItem it = q_item(s, p.ntiles, p.ngh, p.nslot, k);
                const int64_t nst = q_steps(s, it, p.multi, q_rows(s, it, p.multi));
                if (nst == 0) continue;
                const int64_t h0 = it.hg * p.hpi, grp = h0 / (s.H / s.G);
                if (!mbar_wait(bar(RB_QC_EMPTY), (qc_uses & 1) ^ 1, abort_flag, err, 51)) goto producer_end;
                mbar_arrive_expect_tx(bar(RB_QC_FULL), 4 * kBox);
                {
                    const int32_t y = (int32_t)(it.b * s.L + q_t0(s, it, p.multi));
                    for (int kh = 0; kh < 2; ++kh) {
                        tma_load_2d(sbase + kR_Q + kh * kBox, &tmQ, (int32_t)(grp * kN + kh * 64), y, bar(RB_QC_FULL));
                        tma_load_2d(sbase + kR_C + kh * kBox, &tmC, (int32_t)(grp * kN + kh * 64), y, bar(RB_QC_FULL));
                    }
                }
                ++qc_uses;
                qc_loaded = true;
                for (int hp = 0; hp < p.hpi; hp += 2) {
                    for (int64_t j = 0; j < nst; ++j) {
                        if (!mbar_wait(bar(RB_ST_EMPTY + st), ph ^ 1, abort_flag, err, 52)) goto producer_end;
                        mbar_arrive_expect_tx(bar(RB_ST_FULL + st), 2 * kBox);
                        for (int e = 0; e < 2; ++e) {
                            const int32_t y = (int32_t)(((it.b * s.H + h0 + hp + e) * s.M + j) * kN);
                            tma_load_2d(sbase + kR_H + (st * 2 + e) * kBox, &tmH, 0, y, bar(RB_ST_FULL + st));
                        }
                        last_ph[st] = (int)ph;
                        if (++st == kRStages) {
                            st = 0;
                            ph ^= 1;
                        }
                    }
                }
            }
        producer_end:
            for (int q = 0; q < kRStages; ++q)
                if (last_ph[q] >= 0) mbar_drain(bar(RB_ST_FULL + q), (uint32_t)last_ph[q]);
            if (qc_loaded) mbar_drain(bar(RB_QC_FULL), (qc_uses - 1) & 1);
        }
    } else if (warp == 1 || warp == 2) {
        // -------------------------------- MMA ---------------------------------
        // two issuers, lane 0 of warps 1 and 2, take alternate chunk steps (issuer i the steps of U/V buffer
        // i), so that one issues while the other commits and checks its next step's barriers
        setmaxnreg_dec<kRRegsLow>();
        const int issuer = warp - 1;
        if (lane == 0) {
            // A = Q or C (K-major, K = N), B = [dH_h | dH_h+1] (MN-major, K = N), as in the forward
            constexpr uint32_t idesc = idesc_bf16_f32(kTile, 2 * kP, false, true);
            const uint64_t qdesc0 = smem_desc_sw128(sbase + kR_Q, 16, 1024);
            const uint64_t cdesc0 = smem_desc_sw128(sbase + kR_C, 16, 1024);
            uint32_t qc_uses = 0, uv = 0, ph = 0;
            int st = 0;
            bool issued = false;
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const QItem it = q_item(s, p.ntiles, p.ngh, p.nslot, k);
                const int64_t nst = q_steps(s, it, p.multi, q_rows(s, it, p.multi));
                if (nst == 0) continue;
                if (!mbar_wait(bar(RB_QC_FULL), qc_uses & 1, abort_flag, err, 61)) goto mma_end;
                ++qc_uses;
                tc_fence_after();
                for (int hp = 0; hp < p.hpi; hp += 2) {
                    for (int64_t j = 0; j < nst; ++j) {
                        if ((int)(uv & 1) != issuer) {  // the other issuer's step
                            ++uv;
                            if (++st == kRStages) {
                                st = 0;
                                ph ^= 1;
                            }
                            continue;
                        }
                        if (!mbar_wait(bar(RB_ST_FULL + st), ph, abort_flag, err, 62)) goto mma_end;
                        const int ub = uv & 1;  // U and V double-buffered in tensor memory
                        if (!mbar_wait(bar(RB_UV_EMPTY + ub), ((uv >> 1) & 1) ^ 1, abort_flag, err, 63)) goto mma_end;
                        tc_fence_after();
                        const uint64_t bdesc0 = smem_desc_sw128(sbase + kR_H + st * 2 * kBox, kBox, 1024);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t aoff = (uint64_t)((((kk >> 2) * kBox) + (kk & 3) * 32) >> 4);
                            const uint64_t bd = bdesc0 + (uint64_t)((kk * 2048) >> 4);
                            mma_bf16(tmem + ub * 256 + kRT_U, qdesc0 + aoff, bd, idesc, kk > 0);
                            mma_bf16(tmem + ub * 256 + kRT_V, cdesc0 + aoff, bd, idesc, kk > 0);
                        }
                        mma_commit(bar(RB_ST_EMPTY + st));
                        mma_commit(bar(RB_UV_FULL + ub));
                        issued = true;
                        ++uv;
                        if (++st == kRStages) {
                            st = 0;
                            ph ^= 1;
                        }
                    }
                }
                mma_commit(bar(RB_QC_EMPTY));
            }
        mma_end:
            if (issued) {
                const uint32_t done = bar(issuer ? RB_MMA_DONE2 : RB_MMA_DONE);
                mma_commit(done);
                mbar_drain(done, 0);
            }
        }
    } else if (warp < 4) {
        setmaxnreg_dec<kRRegsLow>();  // no role
    } else {
        setmaxnreg_inc<kRRegsHigh>();
        // ------------------------- per-token warps -------------------------
        // warpgroup e = head e of the pair; warp quarter = the tensor-memory lanes (token rows) it owns.
        // Each warp has a 12 KiB staging area: the pair's E, dR hi and dR lo rows come in there (TMA), and
        // dE leaves through it (TMA store).
        const int e = (warp - 4) >> 2, quarter = warp & 3;
        const int row = quarter * 32 + lane;
        constexpr float escale = kLog2e * kRs;
        const uint32_t stg = sbase + kR_STG + (warp - 4) * 12288;
        const uint32_t ldbar = bar(RB_LD + warp - 4);
        const uint32_t lrow = (uint32_t)(quarter * 32) << 16;
        const int L = (int)s.L, H = (int)s.H;
        uint32_t tb = 0, ld_uses = 0;
        bool ld_pending = false;
        float amx = 0.f, emx = 0.f;  // of |a| and of |E_t,p| over this row's pairs: max |a E| <= amx emx
        for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
            const QItem it = q_item(s, p.ntiles, p.ngh, p.nslot, k);
            const int rows = q_rows(s, it, p.multi);
            const int nsteps = (int)q_steps(s, it, p.multi, rows);
            if (nsteps == 0) continue;
            const int t0 = (int)q_t0(s, it, p.multi);
            const int t = t0 + row;
            const int b = (int)it.b;
            const bool valid = row < rows;
            const int my_chunk = valid ? (int)(t / s.S) : 0;  // the row takes the steps j < my_chunk
            for (int hp = 0; hp < p.hpi; hp += 2) {
                const int h = (int)it.hg * p.hpi + hp + e;
                const int eh = p.e_hpg > 1 ? h / p.e_hpg : h;  // the head's E group
                __syncwarp();
                if (lane == 0) {
                    bulk_wait_group_read<0>();  // the last dE stores have read the staging area
                    fence_async_smem_b();
                    mbar_arrive_expect_tx(ldbar, 12288);
                    tma_load_3d(stg, &tmE, eh * kP, t0 + quarter * 32, b, ldbar);
                    tma_load_3d(stg + 4096, &tmDR, h * kP, t0 + quarter * 32, b, ldbar);
                    tma_load_3d(stg + 8192, &tmDR, h * kP + 32, t0 + quarter * 32, b, ldbar);
                }
                ld_pending = true;
                if (!mbar_wait(ldbar, ld_uses & 1, abort_flag, err, 72)) goto tok_end;
                ++ld_uses;
                ld_pending = false;
                // E_t in registers (bf16 pairs); dR_t (fp32, two 32-column halves) stays in the staging area
                uint32_t ev[kP / 2];
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    lds128(stg + lane * 128 + ((q ^ (lane & 7)) << 4), ev[4 * q], ev[4 * q + 1], ev[4 * q + 2],
                           ev[4 * q + 3]);
#pragma unroll
                for (int q = 0; q < kP / 2; ++q) emx = fmaxf(emx, fmaxf(fabsf(bf_lo(ev[q])), fabsf(bf_hi(ev[q]))));
                const uint32_t dr_row = stg + 4096 + lane * 128;  // + half * 4096
                const int64_t hrow = (int64_t)(b * H + h) * L + t;  // [b, h, t] of lse and D
                const float lse2 = valid ? p.lse[hrow] * kLog2e : 0.f;
                const float Dt = valid ? p.D[hrow] : 0.f;
                float *wsc = p.Wsc + (int64_t)(b * H + h) * s.M * L + t;  // [b, h, j, t], j = 0
                float *asc = p.Asc + (int64_t)(b * H + h) * s.M * L + t;
                float dE[kP];
#pragma unroll
                for (int q = 0; q < kP; ++q) dE[q] = 0.f;
                for (int j = 0; j < nsteps; ++j) {
                    const int ub = tb & 1;
                    if (!mbar_wait(bar(RB_UV_FULL + ub), (tb >> 1) & 1, abort_flag, err, 73)) goto tok_end;
                    tc_fence_after();
                    const uint32_t ta = tmem + lrow + ub * 256 + e * kP;
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int half = 0; half < 2; ++half) {  // logit: U . E_t
                        float u[32];
                        tmem_ld_32x32b_x32_after(ta + kRT_U + half * 32, u, acc[0]);
                        tmem_ld_wait_32(u);
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const uint32_t wv = ev[16 * half + q];
                            acc[q & 3] = fmaf(u[2 * q], bf_lo(wv), acc[q & 3]);
                            acc[q & 3] = fmaf(u[2 * q + 1], bf_hi(wv), acc[q & 3]);
                        }
                    }
                    const bool live = j < my_chunk;
                    const float w = live ? exp2f(((acc[0] + acc[1]) + (acc[2] + acc[3])) * escale - lse2) : 0.f;
                    float dacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int half = 0; half < 2; ++half) {  // dw = dR_t . V (fp32 dR)
                        float v[32];
                        tmem_ld_32x32b_x32_after(ta + kRT_V + half * 32, v, dacc[0] + w);
                        uint32_t dr[32];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            lds128(dr_row + half * 4096 + ((q ^ (lane & 7)) << 4), dr[4 * q], dr[4 * q + 1],
                                   dr[4 * q + 2], dr[4 * q + 3]);
                        tmem_ld_wait_32(v);
#pragma unroll
                        for (int q = 0; q < 32; ++q) dacc[q & 3] = fmaf(v[q], __uint_as_float(dr[q]), dacc[q & 3]);
                    }
                    const float a = live ? w * (((dacc[0] + dacc[1]) + (dacc[2] + dacc[3])) - Dt) * kRs : 0.f;
                    amx = fmaxf(amx, fabsf(a));
#pragma unroll
                    for (int half = 0; half < 2; ++half) {  // dE += a U
                        float u[32];
                        tmem_ld_32x32b_x32_after(ta + kRT_U + half * 32, u, a + dE[32 * half]);
                        tmem_ld_wait_32(u);
#pragma unroll
                        for (int q = 0; q < 32; ++q) dE[32 * half + q] = fmaf(a, u[q], dE[32 * half + q]);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(RB_UV_EMPTY + ub));
                    ++tb;
                    if (live) {
                        wsc[(int64_t)j * L] = w;
                        asc[(int64_t)j * L] = a;
                    }
                }
                // dE of the pair out through the staging area (the pair is done with its E and dR rows)
                __syncwarp();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const uint32_t reg = stg + half * 4096;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        sts128(reg + lane * 128 + ((q ^ (lane & 7)) << 4), __float_as_uint(dE[32 * half + 4 * q]),
                               __float_as_uint(dE[32 * half + 4 * q + 1]), __float_as_uint(dE[32 * half + 4 * q + 2]),
                               __float_as_uint(dE[32 * half + 4 * q + 3]));
                    fence_async_smem_b();
                    __syncwarp();
                    if (lane == 0) {
                        // a grouped E: the group's heads add their dE into the (zeroed) group rows
                        if (p.e_hpg > 1)
                            tma_reduce_add_3d(&tmDE, reg, eh * kP + half * 32, t0 + quarter * 32, b);
                        else
                            tma_store_3d(&tmDE, reg, h * kP + half * 32, t0 + quarter * 32, b);
                        bulk_commit_group();
                    }
                }
            }
        }
    tok_end:
        if (ld_pending) mbar_drain(ldbar, ld_uses & 1);
        if (lane == 0) bulk_wait_group<0>();
        amx = warp_max(amx * emx);
        if (p.amax && lane == 0) atomicMax(p.amax, __float_as_uint(amx));
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// gradient GEMM, query side: dQ += (s_a a E) dH16^T / s_a, dC += (s_w w dR) dH16^T / s_w (fp16 rows and
// memories, s_a and s_w the powers of two of pow2_scale); one item = a 128-token tile of one chunk and a
// head group; one step = (head, historical chunk)
// ---------------------------------------------------------------------------
constexpr int kGThreads = 384;  // warp 0 TMA, warp 1 MMA, warps 2-3 idle, warps 4-11 operand builders
// A stage holds one head's chunk memory in fp16; with kKeyRows (the normalised branch's backward) also its
// key rows r (.) dH in fp16, against which the dQ rows are multiplied (dC against the memory itself).
template <bool kKeyRows> struct GqLayout {
    static constexpr int kStages = kKeyRows ? 3 : 4;                       // ring depth
    static constexpr uint32_t kStageBytes = (kKeyRows ? 2 : 1) * kBox;     // [dH] or [dH, K]
    static constexpr uint32_t kH = 0;
    static constexpr uint32_t kOP = kH + kStages * kStageBytes;  // 2 buffers x [E rows, -, R rows, -] boxes
    static constexpr uint32_t kBar = kOP + 8 * kBox;
    static constexpr uint32_t kSmem = kBar + 256 + 1024;
    static_assert(kSmem <= 232448, "gradient kernel exceeds the shared memory of a CTA");
};
constexpr int kGStages = 4;  // the barrier block's room for the deeper ring
constexpr uint32_t kGT_DQ = 0, kGT_DC = 128;

enum { GB_ST_FULL = 0, GB_ST_EMPTY = GB_ST_FULL + kGStages, GB_OP_FULL = GB_ST_EMPTY + kGStages,
       GB_OP_EMPTY = GB_OP_FULL + 2, GB_ACC_FULL = GB_OP_EMPTY + 2, GB_ACC_EMPTY, GB_MMA_DONE, GB_LD,
       GB_COUNT = GB_LD + 8 };
static_assert(GB_COUNT * 8 + 8 <= 256, "barrier block overflows its 256 bytes");

struct BwdGParams {
    Shape s;
    int hpi, ngh, ntiles, multi;
    int64_t nslot, n_items;
    const float *Wsc, *Asc;
    int parts;  // bit 0: dQ (rows a E), bit 1: dC (rows w dR); a part left out builds and multiplies nothing
    const unsigned *amax;  // fp16 rows: max |a E| and max |dR| (float bits), read for the row scales
    int e_hpg;             // heads per E group (E rows of head h are group h / e_hpg); 0 or 1: E per head
};

template <bool kKeyRows>
__global__ void __launch_bounds__(kGThreads, 1)
    k_sma_bwd_gq_tc(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmE,
                    const __grid_constant__ CUtensorMap tmDR, const __grid_constant__ CUtensorMap tmDQ,
                    const __grid_constant__ CUtensorMap tmDC, const BwdGParams p, int *err) {
    using Lay = GqLayout<kKeyRows>;
    constexpr int kGSt = Lay::kStages;
    constexpr uint32_t kG_H = Lay::kH, kG_OP = Lay::kOP, kG_BAR = Lay::kBar;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kG_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kG_BAR + GB_COUNT * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kG_BAR + GB_COUNT * 8 + 4);
    auto bar = [&](int k) { return smem_u32(&bars[k]); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape &s = p.s;
    if (threadIdx.x == 0) {
        for (int q = 0; q < kGSt; ++q) {
            mbar_init(bar(GB_ST_FULL + q), 1);
            mbar_init(bar(GB_ST_EMPTY + q), 1);
        }
        const int nb = 4 * ((p.parts & 1) + ((p.parts >> 1) & 1));  // builder warps of the parts computed
        for (int q = 0; q < 2; ++q) {
            mbar_init(bar(GB_OP_FULL + q), nb);  // every builder warp has written its rows
            mbar_init(bar(GB_OP_EMPTY + q), 1);
        }
        mbar_init(bar(GB_ACC_FULL), 1);
        mbar_init(bar(GB_ACC_EMPTY), nb);
        mbar_init(bar(GB_MMA_DONE), 1);
        for (int w = 0; w < 8; ++w) mbar_init(bar(GB_LD + w), 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmH);
        tma_prefetch_desc(&tmE);
        tma_prefetch_desc(&tmDR);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            uint32_t ph = 0;
            int st = 0;
            int last_ph[kGSt];
            for (int q = 0; q < kGSt; ++q) last_ph[q] = -1;
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const QItem it = q_item(s, p.ntiles, p.ngh, p.nslot, k);
                const int64_t nst = q_steps(s, it, p.multi, q_rows(s, it, p.multi));
                if (nst == 0) continue;
                for (int hh = 0; hh < p.hpi; ++hh) {
                    const int64_t h = it.hg * p.hpi + hh;
                    for (int64_t j = 0; j < nst; ++j) {
                        if (!mbar_wait(bar(GB_ST_EMPTY + st), ph ^ 1, abort_flag, err, 81)) goto producer_end;
                        mbar_arrive_expect_tx(bar(GB_ST_FULL + st), Lay::kStageBytes);
                        const int32_t y = (int32_t)(((it.b * s.H + h) * s.M + j) * kN);
                        const uint32_t slot = sbase + kG_H + st * Lay::kStageBytes;
                        tma_load_2d(slot, &tmH, 0, y, bar(GB_ST_FULL + st));
                        if constexpr (kKeyRows) tma_load_2d(slot + kBox, &tmK, 0, y, bar(GB_ST_FULL + st));
                        last_ph[st] = (int)ph;
                        if (++st == kGSt) {
                            st = 0;
                            ph ^= 1;
                        }
                    }
                }
            }
        producer_end:
            for (int q = 0; q < kGSt; ++q)
                if (last_ph[q] >= 0) mbar_drain(bar(GB_ST_FULL + q), (uint32_t)last_ph[q]);
        }
    } else if (warp == 1) {
        // -------------------------------- MMA ---------------------------------
        if (lane == 0) {
            // A = operand rows (K-major, fp16), B = dH (or the key rows) read with K = P (K-major), M =
            // tokens, N = n
            constexpr uint32_t idesc = idesc_f32acc(kTile, kN, false, false, true);
            constexpr int kKSteps = 4;
            uint32_t u = 0, ph = 0, items = 0;
            int st = 0;
            bool issued = false;
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const QItem it = q_item(s, p.ntiles, p.ngh, p.nslot, k);
                const int64_t nst = q_steps(s, it, p.multi, q_rows(s, it, p.multi));
                if (nst == 0) continue;
                if (!mbar_wait(bar(GB_ACC_EMPTY), (items & 1) ^ 1, abort_flag, err, 82)) goto mma_end;
                bool first = true;
                for (int hh = 0; hh < p.hpi; ++hh) {
                    for (int64_t j = 0; j < nst; ++j, ++u) {
                        const int buf = u & 1;
                        if (!mbar_wait(bar(GB_ST_FULL + st), ph, abort_flag, err, 83)) goto mma_end;
                        if (!mbar_wait(bar(GB_OP_FULL + buf), (u >> 1) & 1, abort_flag, err, 84)) goto mma_end;
                        tc_fence_after();
                        const uint32_t slot = sbase + kG_H + st * Lay::kStageBytes;
                        const uint64_t bd = smem_desc_sw128(slot, 16, 1024);
                        const uint32_t ob = sbase + kG_OP + buf * 4 * kBox;
                        const uint64_t kd = kKeyRows ? smem_desc_sw128(slot + kBox, 16, 1024) : bd;  // dQ's B
#pragma unroll
                        for (int kk = 0; kk < kKSteps; ++kk) {
                            const uint64_t ae = smem_desc_sw128(ob + kk * 32, 16, 1024);
                            const uint64_t ar = smem_desc_sw128(ob + 2 * kBox + kk * 32, 16, 1024);
                            const uint64_t boff = (uint64_t)((kk * 32) >> 4);
                            const uint32_t acc = (first && kk == 0) ? 0u : 1u;
                            if (p.parts & 1) mma_bf16(tmem + kGT_DQ, ae, kd + boff, idesc, acc);
                            if (p.parts & 2) mma_bf16(tmem + kGT_DC, ar, bd + boff, idesc, acc);
                        }
                        first = false;
                        mma_commit(bar(GB_OP_EMPTY + buf));
                        mma_commit(bar(GB_ST_EMPTY + st));
                        issued = true;
                        if (++st == kGSt) {
                            st = 0;
                            ph ^= 1;
                        }
                    }
                }
                mma_commit(bar(GB_ACC_FULL));
                ++items;
            }
        mma_end:
            if (issued) {
                mma_commit(bar(GB_MMA_DONE));
                mbar_drain(bar(GB_MMA_DONE), 0);
            }
        }
    } else if (warp >= 4) {
        // ------------------------- operand builders -------------------------
        // warpgroup 0 writes the rows a_tj E_t (for dQ), warpgroup 1 the rows w_tj dR_t (for dC), in fp16,
        // into the step's buffer; warp quarter = the 32 token rows it owns. A head's E (or dR) rows arrive by
        // TMA in boxes the fp16 operands leave free, one head ahead (issued as soon as the current head's
        // rows are in registers). At the end of an item dQ (or dC) leaves through the part's first box of
        // the two buffers.
        const int e = (warp - 4) >> 2, quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t ldbar = bar(GB_LD + warp - 4);
        const uint32_t lrow = (uint32_t)(quarter * 32) << 16;
        const int L = (int)s.L, H = (int)s.H;
        const float *scal = e ? p.Wsc : p.Asc;
        const float sig = pow2_scale(p.amax[e]);  // fp16 rows: |sig x| < 2^14
        const float inv_sig = 1.f / sig;
        uint32_t u = 0, ld_uses = 0, acc_uses = 0;
        bool ld_pending = false;
        const int64_t n_my_items = ((p.parts >> e) & 1) ? p.n_items : 0;  // a part left out: no work
        // fp16: the staging boxes of the next head's rows (E: box 1 of buffer 0; dR: box 3 of buffers 0, 1)
        const uint32_t stg = sbase + kG_OP + (e ? 3 : 1) * kBox + quarter * 4096;
        auto live_item = [&](int64_t k2) {  // the first item at or after k2 (in this CTA's order) with steps
            while (k2 < n_my_items) {
                const QItem i2 = q_item(s, p.ntiles, p.ngh, p.nslot, k2);
                if (q_steps(s, i2, p.multi, q_rows(s, i2, p.multi)) > 0) break;
                k2 = sched_next(k2);
            }
            return k2;
        };
        auto issue_rows = [&](int64_t k2, int hh2) {  // fp16: head hh2 of item k2's rows into the staging boxes
            const QItem i2 = q_item(s, p.ntiles, p.ngh, p.nslot, k2);
            const int32_t h2 = (int32_t)(i2.hg * p.hpi + hh2), ty = (int32_t)(q_t0(s, i2, p.multi) + quarter * 32);
            __syncwarp();  // every lane has read the boxes' previous rows
            if (lane == 0) {
                fence_async_smem_b();
                mbar_arrive_expect_tx(ldbar, e ? 8192 : 4096);
                if (e == 0) {
                    tma_load_3d(stg, &tmE, (p.e_hpg > 1 ? h2 / p.e_hpg : h2) * kP, ty, (int32_t)i2.b, ldbar);
                } else {  // dR in fp32: columns 0-31 and 32-63
                    tma_load_3d(stg, &tmDR, h2 * kP, ty, (int32_t)i2.b, ldbar);
                    tma_load_3d(stg + 4 * kBox, &tmDR, h2 * kP + 32, ty, (int32_t)i2.b, ldbar);
                }
            }
            ld_pending = true;
        };
        {
            const int64_t k0 = live_item(blockIdx.x);
            if (k0 < n_my_items) issue_rows(k0, 0);
        }
        for (int64_t k = blockIdx.x; k < n_my_items; k = sched_next(k)) {
            const QItem it = q_item(s, p.ntiles, p.ngh, p.nslot, k);
            const int rows = q_rows(s, it, p.multi);
            const int nsteps = (int)q_steps(s, it, p.multi, rows);
            if (nsteps == 0) continue;
            const int t0 = (int)q_t0(s, it, p.multi);
            const int t = t0 + row;
            const int b = (int)it.b;
            const bool valid = row < rows;
            const int my_chunk = valid ? (int)(t / s.S) : 0;  // the row takes the steps j < my_chunk
            const int grp = (int)(it.hg * p.hpi / (s.H / s.G));
            for (int hh = 0; hh < p.hpi; ++hh) {
                const int h = (int)it.hg * p.hpi + hh;
                const uint32_t hi0 = stg, half_stride = 4 * kBox;  // dR's second 32 columns: box 3 of buffer 1
                if (!mbar_wait(ldbar, ld_uses & 1, abort_flag, err, 92)) goto g_end;
                ++ld_uses;
                ld_pending = false;
                float val[kP];  // E_t or dR_t of this row, fp32
                if (e == 0) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint32_t x[4];
                        lds128(hi0 + lane * 128 + ((q ^ (lane & 7)) << 4), x[0], x[1], x[2], x[3]);
#pragma unroll
                        for (int w4 = 0; w4 < 4; ++w4) {
                            val[8 * q + 2 * w4] = bf_lo(x[w4]);
                            val[8 * q + 2 * w4 + 1] = bf_hi(x[w4]);
                        }
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        uint32_t x[4];
                        lds128(hi0 + (q >> 3) * half_stride + lane * 128 + (((q & 7) ^ (lane & 7)) << 4), x[0], x[1],
                               x[2], x[3]);
#pragma unroll
                        for (int w4 = 0; w4 < 4; ++w4) val[4 * q + w4] = __uint_as_float(x[w4]);
                    }
                }
                if (hh + 1 < p.hpi) {  // the next head's rows, while this head's steps run
                    issue_rows(k, hh + 1);
                } else {
                    const int64_t k2 = live_item(sched_next(k));
                    if (k2 < n_my_items) issue_rows(k2, 0);
                }
                const float *sc_row = scal + (int64_t)(b * H + h) * s.M * L + t;  // [b, h, j, t], j = 0
                float sc_next = my_chunk > 0 ? __ldg(sc_row) : 0.f;  // one step ahead, so its latency overlaps a build
                for (int j = 0; j < nsteps; ++j, ++u) {
                    const int buf = u & 1;
                    const float sc = sc_next;
                    sc_next = j + 1 < my_chunk ? __ldg(sc_row + (int64_t)(j + 1) * L) : 0.f;
                    if (!mbar_wait(bar(GB_OP_EMPTY + buf), ((u >> 1) & 1) ^ 1, abort_flag, err, 93)) goto g_end;
                    const uint32_t hi = sbase + kG_OP + buf * 4 * kBox + (2 * e) * kBox + quarter * 4096;
                    const float f = sc * sig;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint32_t o[4];
#pragma unroll
                        for (int w4 = 0; w4 < 4; ++w4)
                            o[w4] = pack_f16x2(f * val[8 * q + 2 * w4], f * val[8 * q + 2 * w4 + 1]);
                        sts128(hi + lane * 128 + ((q ^ (lane & 7)) << 4), o[0], o[1], o[2], o[3]);
                    }
                    fence_async_smem_b();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(GB_OP_FULL + buf));
                }
            }
            // dQ (warpgroup 0) or dC (warpgroup 1) of the item through this warp's rows of buffer 0, added
            // into the output (zeroed by the host): the items of the other head groups that share the Q/C
            // group add theirs to the same rows
            if (!mbar_wait(bar(GB_ACC_FULL), acc_uses & 1, abort_flag, err, 94)) goto g_end;
            ++acc_uses;
            tc_fence_after();
#pragma unroll 1
            for (int c4 = 0; c4 < 4; ++c4) {
                const uint32_t reg = sbase + kG_OP + (c4 & 1) * 4 * kBox + (2 * e) * kBox + quarter * 4096;
                if (lane == 0) bulk_wait_group_read<1>();
                __syncwarp();
                float v[32];
                tmem_ld_32x32b_x32(tmem + lrow + (e ? kGT_DC : kGT_DQ) + c4 * 32, v);
                tmem_ld_wait_32(v);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    sts128(reg + lane * 128 + ((q ^ (lane & 7)) << 4), __float_as_uint(v[4 * q] * inv_sig),
                           __float_as_uint(v[4 * q + 1] * inv_sig), __float_as_uint(v[4 * q + 2] * inv_sig),
                           __float_as_uint(v[4 * q + 3] * inv_sig));
                fence_async_smem_b();
                __syncwarp();
                if (lane == 0) {
                    tma_reduce_add_3d(e ? &tmDC : &tmDQ, reg, grp * kN + c4 * 32, t0 + quarter * 32, b);
                    bulk_commit_group();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(GB_ACC_EMPTY));
                bulk_wait_group_read<0>();  // the staging boxes are free again before the next item builds
            }
            __syncwarp();
        }
    g_end:
        if (ld_pending) mbar_drain(ldbar, ld_uses & 1);
        if (lane == 0) bulk_wait_group<0>();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------------------
// gradient GEMM, memory side: [ddH_c | ddH_c+1] += Q_T^T [aE_c | aE_c+1] + C_T^T [w dR_c | w dR_c+1]
// one item = one head and a block of 8 chunk memories; it streams the 128-token tiles after the block's
// first chunk. Per tile the steps run part by part: first every chunk pair's key term (A = the Q tile), then
// every pair's value term (A = the C tile), so that each tile is free once its part's last product is done
// and the next tile's Q loads while the value terms run (and its C while the next key terms run).
// Warpgroup 0 builds the key rows a E_t, warpgroup 1 the value rows w dR_t, each for both chunks of a pair;
// a warpgroup loads its next tile's row and scalars right after its last step of a tile, so that the loads
// land while the other warpgroup's steps run. Q and C come as fp16 copies and the rows are rounded to fp16
// after one power-of-two scale s (the smaller of the two parts' scales when both are summed); K = 128 tokens,
// the accumulators divided by s.
// ---------------------------------------------------------------------------
constexpr int kMBlock = 8;                   // chunk memories per item (4 pairs x 128 tensor-memory columns)
// Shared memory: the Q tile (2 boxes), the C tile (2 boxes) and four operand buffers of [c, c+1] (128 KiB).
// The output leaves through the first four boxes of the operand buffers.
struct GmLayout {
    static constexpr int kBufs = 4;
    static constexpr uint32_t kBufBoxes = 2;
    static constexpr uint32_t kQ = 0, kC = 2 * kBox;
    static constexpr uint32_t kOP = 4 * kBox;
    static constexpr uint32_t kBar = kOP + kBufs * kBufBoxes * kBox;
    static constexpr uint32_t kSmem = kBar + 256 + 1024;
    static_assert(kSmem <= 232448, "memory-side kernel exceeds the shared memory of a CTA");
};

enum { MB_T_FULL = 0, MB_T_EMPTY = MB_T_FULL + 2, MB_OP_FULL = MB_T_EMPTY + 2, MB_OP_EMPTY = MB_OP_FULL + 4,
       MB_ACC_FULL = MB_OP_EMPTY + 4, MB_ACC_EMPTY, MB_MMA_DONE, MB_COUNT };  // MB_T_*: [Q, C]
static_assert(MB_COUNT * 8 + 8 <= 256, "barrier block overflows its 256 bytes");

struct BwdMParams {
    Shape s;
    int nblk;          // chunk blocks per (b, h)
    int64_t nslots;    // 128-token tiles of a batch row
    int64_t n_items;   // nblk * Bt * H
    const __nv_bfloat16 *E;
    const float *dR;
    const float *Wsc, *Asc;
    int parts;  // bit 0: the key term Q^T (a E), bit 1: the value term C^T (w dR)
    const unsigned *amax;  // fp16 rows: max |a E| and max |dR| (float bits), read for the row scale
    int key_amax;          // the word of amax that bounds the key rows (0; 2 in the normalised branch)
    int e_hpg;             // heads per E group (E rows of head h are group h / e_hpg); 0 or 1: E per head
};

struct MItem {
    int b, h, c_lo, c_hi;  // chunk memories [c_lo, c_hi) of head h, batch row b
};

__device__ __forceinline__ MItem m_item(const BwdMParams &p, int64_t k) {
    const int64_t bh = p.s.Bt * p.s.H;
    MItem it;
    const int cb = (int)(k / bh);  // block 0 (the most later tiles) first
    const int r = (int)(k - (int64_t)cb * bh);
    it.b = r / (int)p.s.H;
    it.h = r - it.b * (int)p.s.H;
    it.c_lo = cb * kMBlock;
    it.c_hi = min(it.c_lo + kMBlock, (int)p.s.M - 1);
    return it;
}

// rows of the batch row's 128-token tile g (a tile of one chunk for S >= 128, of 128 / S chunks below)
__device__ __forceinline__ int m_rows(const BwdMParams &p, int64_t g) {
    return (int)max((int64_t)0, min((int64_t)kTile, p.s.L - g * kTile));
}

// the first tile with a token after the item's first chunk memory
__device__ __forceinline__ int64_t m_first(const BwdMParams &p, const MItem &it) {
    return (int64_t)(it.c_lo + 1) * p.s.S / kTile;
}

// chunk of the last row of tile g (rows > 0)
__device__ __forceinline__ int64_t m_last_chunk(const BwdMParams &p, int64_t g, int rows) {
    return (g * kTile + rows - 1) / p.s.S;
}

// chunk pairs of item `it` that a tile whose last row is in chunk i contributes to
__device__ __forceinline__ int m_pairs(const MItem &it, int64_t i) {
    const int top = (int)min((int64_t)it.c_hi, i);
    return top > it.c_lo ? (top - it.c_lo + 1) / 2 : 0;
}

__global__ void __launch_bounds__(kGThreads, 1)
    k_sma_bwd_gm_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC,
                    const __grid_constant__ CUtensorMap tmDDH, const BwdMParams p, int *err) {
    using Lay = GmLayout;
    constexpr int kNB = Lay::kBufs;
    constexpr uint32_t kBufBytes = Lay::kBufBoxes * kBox;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Lay::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Lay::kBar + MB_COUNT * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Lay::kBar + MB_COUNT * 8 + 4);
    auto bar = [&](int k) { return smem_u32(&bars[k]); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape &s = p.s;
    const int64_t ntot = p.nslots;  // tiles of a batch row
    if (threadIdx.x == 0) {
        for (int q = 0; q < 2; ++q) {
            mbar_init(bar(MB_T_FULL + q), 1);
            mbar_init(bar(MB_T_EMPTY + q), 1);
        }
        for (int q = 0; q < kNB; ++q) {
            mbar_init(bar(MB_OP_FULL + q), 4);  // the four warps of the part's warpgroup
            mbar_init(bar(MB_OP_EMPTY + q), 1);
        }
        mbar_init(bar(MB_ACC_FULL), 1);
        mbar_init(bar(MB_ACC_EMPTY), 8);  // every builder warp has read its accumulators and staged them out
        mbar_init(bar(MB_MMA_DONE), 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------ producer: Q and C tiles ------------------------------
        if (lane == 0) {
            uint32_t uses[2] = {0, 0};
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const MItem it = m_item(p, k);
                const int64_t grp = it.h / (s.H / s.G);
                for (int64_t g = m_first(p, it); g < ntot; ++g) {
                    if (m_rows(p, g) == 0) continue;
                    const int32_t y = (int32_t)(it.b * s.L + g * kTile);
                    for (int part = 0; part < 2; ++part) {
                        if (!((p.parts >> part) & 1)) continue;
                        if (!mbar_wait(bar(MB_T_EMPTY + part), (uses[part] & 1) ^ 1, abort_flag, err, 101))
                            goto producer_end;
                        mbar_arrive_expect_tx(bar(MB_T_FULL + part), 2 * kBox);
                        const uint32_t dst = sbase + (part ? Lay::kC : Lay::kQ);
                        for (int kh = 0; kh < 2; ++kh)
                            tma_load_2d(dst + kh * kBox, part ? &tmC : &tmQ, (int32_t)(grp * kN + kh * 64), y,
                                        bar(MB_T_FULL + part));
                        ++uses[part];
                    }
                }
            }
        producer_end:
            for (int part = 0; part < 2; ++part)
                if (uses[part]) mbar_drain(bar(MB_T_FULL + part), (uses[part] - 1) & 1);
        }
    } else if (warp == 1) {
        // -------------------------------- MMA ---------------------------------
        if (lane == 0) {
            // A = Q_T^T or C_T^T (MN-major: M = n over the tile's two boxes, K = tokens),
            // B = [X_c | X_c+1] (MN-major: N = p over the two chunks' boxes, K = tokens), fp16
            constexpr uint32_t idesc = idesc_f32acc(kN, 2 * kP, true, true, true);
            constexpr int kKSteps = 8;
            uint32_t tu[2] = {0, 0}, u = 0, items = 0;
            bool issued = false;
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const MItem it = m_item(p, k);
                if (!mbar_wait(bar(MB_ACC_EMPTY), (items & 1) ^ 1, abort_flag, err, 102)) goto mma_end;
                uint32_t started = 0;  // chunk pairs whose accumulator holds this item's sum
                for (int64_t g = m_first(p, it); g < ntot; ++g) {
                    const int rows = m_rows(p, g);
                    if (rows == 0) continue;
                    const int np = m_pairs(it, m_last_chunk(p, g, rows));
                    for (int part = 0; part < 2; ++part) {  // part 0: Q with a E; part 1: C with w dR
                        if (!((p.parts >> part) & 1)) continue;
                        if (!mbar_wait(bar(MB_T_FULL + part), tu[part] & 1, abort_flag, err, 103)) goto mma_end;
                        ++tu[part];
                        const uint32_t ab = sbase + (part ? Lay::kC : Lay::kQ);
                        for (int cp = 0; cp < np; ++cp) {
                            const uint32_t uu = u++;
                            const int buf = (int)(uu % kNB);
                            if (!mbar_wait(bar(MB_OP_FULL + buf), (uu / kNB) & 1, abort_flag, err, 104)) goto mma_end;
                            tc_fence_after();
                            const uint32_t ob = sbase + Lay::kOP + buf * kBufBytes;
#pragma unroll
                            for (int kk = 0; kk < kKSteps; ++kk) {
                                const uint64_t ad = smem_desc_sw128(ab + (kk & 7) * 2048, kBox, 1024);
                                const uint64_t bd = smem_desc_sw128(ob + kk * 2048, kBox, 1024);
                                const uint32_t acc = (kk == 0 && !(started >> cp & 1)) ? 0u : 1u;
                                mma_bf16(tmem + cp * 128, ad, bd, idesc, acc);
                            }
                            started |= 1u << cp;
                            mma_commit(bar(MB_OP_EMPTY + buf));
                            issued = true;
                        }
                        mma_commit(bar(MB_T_EMPTY + part));  // the part's products of this tile are issued
                    }
                }
                mma_commit(bar(MB_ACC_FULL));
                ++items;
            }
        mma_end:
            if (issued) {
                mma_commit(bar(MB_MMA_DONE));
                mbar_drain(bar(MB_MMA_DONE), 0);
            }
        }
    } else if (warp >= 4) {
        // ------------------------- operand builders -------------------------
        // warpgroup e builds part e (0: rows a E_t against Q, 1: rows w dR_t against C) for both chunks of
        // every pair; warp quarter = the 32 token rows it owns. A thread keeps one tile's row (E as bf16 pairs,
        // or dR in fp32) and the tile's scalars of the block's chunks; the next tile's are loaded into the same
        // registers right after the thread's last step of a tile.
        const int e = (warp - 4) >> 2, quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lrow = (uint32_t)(quarter * 32) << 16;
        const int L = (int)s.L, H = (int)s.H;
        const bool mine = ((p.parts >> e) & 1) != 0;  // this warpgroup's part is computed
        // fp16 rows: |sig x| < 2^14 for the parts summed into the accumulators
        const float sa = pow2_scale(p.amax[p.key_amax]), sw = pow2_scale(p.amax[1]);
        const float sig = p.parts == 1 ? sa : (p.parts == 2 ? sw : fminf(sa, sw));
        const float inv_sig = 1.f / sig;
        const float *scp = e ? p.Wsc : p.Asc;
        uint32_t u = 0, acc_uses = 0;
        uint32_t rv[kP];    // the row: E_t as bf16 pairs in rv[0..31] (warpgroup 0), dR_t as fp32 bits (1)
        float sc[kMBlock];  // the tile's scalar of each chunk of the block (0 past the row's history)
        // the row data and scalars of tile g of item `it` into ev / dv and sc
        auto load_tile = [&](const MItem &it, int64_t g) {
            const int rows = m_rows(p, g);
            const int t = (int)(g * kTile) + row;
            const bool valid = row < rows;
            const int i = valid ? (int)(t / s.S) : 0;  // this row's chunk: it feeds memories c < i
            const int64_t ro = ((int64_t)(it.b * L + (valid ? t : 0)) * H + it.h) * kP;
            if (e == 0) {
                const int64_t reo = p.e_hpg > 1  // E row of the head's group: [Bt, L, H / e_hpg, P]
                                        ? ((int64_t)(it.b * L + (valid ? t : 0)) * (H / p.e_hpg) + it.h / p.e_hpg) * kP
                                        : ro;
                const uint4 *pe = reinterpret_cast<const uint4 *>(p.E + reo);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint4 a = valid ? __ldg(pe + q) : make_uint4(0u, 0u, 0u, 0u);
                    rv[4 * q] = a.x, rv[4 * q + 1] = a.y, rv[4 * q + 2] = a.z, rv[4 * q + 3] = a.w;
                }
            } else {
                const uint4 *pr = reinterpret_cast<const uint4 *>(p.dR + ro);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const uint4 r = valid ? __ldg(pr + q) : make_uint4(0u, 0u, 0u, 0u);
                    rv[4 * q] = r.x, rv[4 * q + 1] = r.y, rv[4 * q + 2] = r.z, rv[4 * q + 3] = r.w;
                }
            }
            const int top = min(it.c_hi, i);
#pragma unroll
            for (int q = 0; q < kMBlock; ++q) {
                const int c = it.c_lo + q;
                const int64_t si = ((int64_t)(it.b * H + it.h) * s.M + c) * L + t;
                sc[q] = (valid && c < top) ? __ldg(scp + si) : 0.f;
            }
        };
        // the first tile of the first item
        int64_t k = blockIdx.x;
        int64_t g = k < p.n_items ? m_first(p, m_item(p, k)) : 0;
        auto next_live = [&](int64_t &k2, int64_t &g2) {  // advance (k2, g2) to a tile with rows, or k2 = end
            while (k2 < p.n_items) {
                const MItem it2 = m_item(p, k2);
                while (g2 < ntot && m_rows(p, g2) == 0) ++g2;
                if (g2 < ntot) return;
                k2 = sched_next(k2);
                if (k2 < p.n_items) g2 = m_first(p, m_item(p, k2));
                (void)it2;
            }
        };
        next_live(k, g);
        if (mine && k < p.n_items) load_tile(m_item(p, k), g);
        for (; k < p.n_items; k = sched_next(k)) {
            const MItem it = m_item(p, k);
            // every builder warp has finished the previous item's epilogue (its staging boxes are the
            // operand buffers this item's first steps write)
            if (acc_uses > 0 && !mbar_wait(bar(MB_ACC_EMPTY), (acc_uses - 1) & 1, abort_flag, err, 113)) goto m_end;
            for (g = m_first(p, it); g < ntot; ++g) {
                const int rows = m_rows(p, g);
                if (rows == 0) continue;
                const int np = m_pairs(it, m_last_chunk(p, g, rows));
                // the other part's steps of this tile come before (value part) or after (key part) this one's
                if (e == 1 && (p.parts & 1)) u += np;
                if (mine) {
                    for (int cp = 0; cp < np; ++cp) {
                        const uint32_t uu = u++;
                        const int buf = (int)(uu % kNB);
                        if (!mbar_wait(bar(MB_OP_EMPTY + buf), ((uu / kNB) & 1) ^ 1, abort_flag, err, 111)) goto m_end;
                        const uint32_t ob = sbase + Lay::kOP + buf * kBufBytes + quarter * 4096;
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch) {  // chunks c_lo + 2 cp + ch
                            float scv = 0.f;
#pragma unroll
                            for (int q = 0; q < kMBlock; ++q)
                                if (q == 2 * cp + ch) scv = sc[q];
                            const uint32_t hi = ob + ch * kBox;
                            const float f = scv * sig;
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                uint32_t o[4];
#pragma unroll
                                for (int w4 = 0; w4 < 4; ++w4) {
                                    const int kx = 8 * q + 2 * w4;
                                    const float x0 = e ? __uint_as_float(rv[kx]) : bf_lo(rv[kx / 2]);
                                    const float x1 = e ? __uint_as_float(rv[kx + 1]) : bf_hi(rv[kx / 2]);
                                    o[w4] = pack_f16x2(f * x0, f * x1);
                                }
                                sts128(hi + lane * 128 + ((q ^ (lane & 7)) << 4), o[0], o[1], o[2], o[3]);
                            }
                        }
                        fence_async_smem_b();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(MB_OP_FULL + buf));
                    }
                    // the next tile's row and scalars, while the other warpgroup's steps run
                    int64_t k2 = k, g2 = g + 1;
                    next_live(k2, g2);
                    if (k2 < p.n_items) load_tile(m_item(p, k2), g2);
                }
                if (e == 0 && (p.parts & 2)) u += np;
            }
            // ddH of the item's chunk memories (chunk c_lo + 2 cp + e of every pair) through the first four
            // boxes of the operand buffers
            if (!mbar_wait(bar(MB_ACC_FULL), acc_uses & 1, abort_flag, err, 112)) goto m_end;
            ++acc_uses;
            tc_fence_after();
            for (int cp = 0; 2 * cp < it.c_hi - it.c_lo; ++cp) {
                const int c = it.c_lo + 2 * cp + e;
                if (c >= it.c_hi) continue;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    const uint32_t reg = sbase + Lay::kOP + (e + 2 * half) * kBox + quarter * 4096;
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                    float v[32];
                    tmem_ld_32x32b_x32(tmem + lrow + cp * 128 + e * kP + half * 32, v);
                    tmem_ld_wait_32(v);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        sts128(reg + lane * 128 + ((q ^ (lane & 7)) << 4), __float_as_uint(v[4 * q] * inv_sig),
                               __float_as_uint(v[4 * q + 1] * inv_sig), __float_as_uint(v[4 * q + 2] * inv_sig),
                               __float_as_uint(v[4 * q + 3] * inv_sig));
                    fence_async_smem_b();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(&tmDDH, reg, half * 32,
                                     (int32_t)(((int64_t)(it.b * H + it.h) * s.M + c) * kN + quarter * 32), 0);
                        bulk_commit_group();
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                bulk_wait_group_read<0>();  // the stores have read the staging boxes
                mbar_arrive(bar(MB_ACC_EMPTY));
            }
            __syncwarp();
        }
    m_end:
        if (lane == 0) bulk_wait_group<0>();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// Backward of the normalised score branch (App. B.1 eq 25-27) on the tensor cores.
//
// With Qb = iq Q_t, Eb = ie E_t (RMSNorm, unit weight) and the key rows Kr[c] = diag(r_c) dH[c],
// r_{c,n} = (mean_p dH[c]_{n,p}^2 + eps)^(-1/2), the forward's logit is l = Qb Kr[c] Eb / sqrt(N) and its
// value C_t dH[c]. Per token t, head h and chunk c < chunk(t), with U = Qb Kr[c] (a P-vector):
//   w = exp(l - lse_t), dw = dR_t . (C_t dH[c]), D_t = sum_c w dw, a = w (dw - D_t) / sqrt(N),
//   dEb += a U, dQb += a Kr[c] Eb, dC += w dH[c] dR_t,
//   ddH[c] += C_t^T (w dR_t) + diag(r_c) G - diag(r_c^3 rho_c / P) dH[c],  G = Qb^T (a Eb),
//   rho_{c,n} = sum_p G_{n,p} dH[c]_{n,p}  (the derivative of r_{c,n} through its row),
// then dQ = iq dQb - iq^3 Q (Q . dQb) / N and dE = ie dEb - ie^3 E (E . dEb) / P.
//
// The logits decide the weights, and a sharp softmax amplifies their error in the heavy-tailed dQ and dE:
// keys rounded once to fp16 moved dQ by 2.4-4.9e-2 of its rms (float64 emulation). So the key rows enter
// the tensor cores as a bf16 pair Kr = Khi + Klo (16 significant bits), made once per chunk memory row by
// k_norm_key_rows, and U = iq (Q Khi + Q Klo). The statistics lse and D are recomputed from these logits
// (a first pass of k_sma_bwd_rn_tc), so that the weights do not depend on the forward's precision.
// The gradient GEMMs then run on the plain backward's kernels, in fp16 as there: dC (rows w dR against dH),
// dQb (rows a ie E against the key rows r (.) dH), G (rows a iq ie E against Q) and C^T (w dR), each set of
// rows after its own power-of-two scale (the second recompute pass finds the maxima); k_norm_ddh_combine
// and k_norm_dq_post apply the r and RMSNorm factors.
// ---------------------------------------------------------------------------

// r, Khi and Klo of every chunk memory row (8 lanes a 128-byte row), eps inside the mean; and for the gradient
// GEMMs the key rows r (.) dH and the memory itself in fp16 (a memory value of 65536 or more raises
// kRangeBwdOperands: fp16 cannot hold it)
__global__ void __launch_bounds__(256) k_norm_key_rows(const __nv_bfloat16 *__restrict__ dH, float *__restrict__ r,
                                                       __nv_bfloat16 *__restrict__ khi, __nv_bfloat16 *__restrict__ klo,
                                                       uint4 *__restrict__ k16, uint4 *__restrict__ dh16, int *range,
                                                       int64_t rows, float eps) {
    const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = gt >> 3;
    const int part = threadIdx.x & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row < rows) v = __ldg(reinterpret_cast<const uint4 *>(dH + row * kP) + part);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float sq = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) sq = fmaf(bf_lo(w[u]), bf_lo(w[u]), fmaf(bf_hi(w[u]), bf_hi(w[u]), sq));
    sq += __shfl_xor_sync(0xffffffffu, sq, 4);
    sq += __shfl_xor_sync(0xffffffffu, sq, 2);
    sq += __shfl_xor_sync(0xffffffffu, sq, 1);
    const float rr = rsqrtf(sq * (1.f / kP) + eps);
    if (row >= rows) return;
    if (part == 0) r[row] = rr;
    uint32_t oh[4], ol[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) split_bf16x2(bf_lo(w[u]) * rr, bf_hi(w[u]) * rr, oh[u], ol[u]);
    reinterpret_cast<uint4 *>(khi + row * kP)[part] = make_uint4(oh[0], oh[1], oh[2], oh[3]);
    reinterpret_cast<uint4 *>(klo + row * kP)[part] = make_uint4(ol[0], ol[1], ol[2], ol[3]);
    uint32_t ok[4], od[4];
    bool over = false;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        ok[u] = pack_f16x2(bf_lo(w[u]) * rr, bf_hi(w[u]) * rr);
        od[u] = pack_f16x2(bf_lo(w[u]), bf_hi(w[u]));
        over |= (w[u] & 0x7fffu) >= 0x4780u || (w[u] & 0x7fff0000u) >= 0x47800000u;
    }
    k16[row * (kP / 8) + part] = make_uint4(ok[0], ok[1], ok[2], ok[3]);
    dh16[row * (kP / 8) + part] = make_uint4(od[0], od[1], od[2], od[3]);
    if (over && range) atomicOr(range, kRangeBwdOperands);
}

// iq = (mean_n Q_t^2 + eps)^(-1/2) of every (b, t, g) row of Q (16 lanes a 256-byte row)
__global__ void __launch_bounds__(256) k_norm_q_rms(const __nv_bfloat16 *__restrict__ Q, float *__restrict__ iq,
                                                    int64_t rows, float eps) {
    const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = gt >> 4;
    const int part = threadIdx.x & 15;
    float sq = 0.f;
    if (row < rows) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(Q + row * kN) + part);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) sq = fmaf(bf_lo(w[u]), bf_lo(w[u]), fmaf(bf_hi(w[u]), bf_hi(w[u]), sq));
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if (row < rows && part == 0) iq[row] = rsqrtf(sq * (1.f / kN) + eps);
}

// dQ = iq dQb - iq^3 Q (Q . dQb) / N per (b, t, g) row (16 lanes a row of 128 floats)
__global__ void __launch_bounds__(256) k_norm_dq_post(const __nv_bfloat16 *__restrict__ Q, const float *__restrict__ iq,
                                                      const float *__restrict__ dqb, float *__restrict__ dQ, int64_t rows) {
    const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = gt >> 4;
    const int part = threadIdx.x & 15;
    float q[8], g[8], dot = 0.f;
    if (row < rows) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(Q + row * kN) + part);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) q[2 * u] = bf_lo(w[u]), q[2 * u + 1] = bf_hi(w[u]);
        const float4 a = __ldg(reinterpret_cast<const float4 *>(dqb + row * kN) + 2 * part);
        const float4 b = __ldg(reinterpret_cast<const float4 *>(dqb + row * kN) + 2 * part + 1);
        g[0] = a.x, g[1] = a.y, g[2] = a.z, g[3] = a.w, g[4] = b.x, g[5] = b.y, g[6] = b.z, g[7] = b.w;
#pragma unroll
        for (int u = 0; u < 8; ++u) dot = fmaf(q[u], g[u], dot);
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    if (row >= rows) return;
    const float f = iq[row], f3 = f * f * f * dot * (1.f / kN);
    float o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) o[u] = fmaf(f, g[u], -f3 * q[u]);
    reinterpret_cast<float4 *>(dQ + row * kN)[2 * part] = make_float4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<float4 *>(dQ + row * kN)[2 * part + 1] = make_float4(o[4], o[5], o[6], o[7]);
}

// ddH = GV + r G - r^3 rho dH / P per chunk memory row, rho = G . dH[row]; G is read from (and the result
// written over) ddH (16 lanes a row of 64 floats, 4 each)
__global__ void __launch_bounds__(256) k_norm_ddh_combine(const __nv_bfloat16 *__restrict__ dH, const float *__restrict__ r,
                                                          const float *__restrict__ gv, float *__restrict__ ddH,
                                                          int64_t rows) {
    const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = gt >> 4;
    const int part = threadIdx.x & 15;
    float d[4] = {0.f, 0.f, 0.f, 0.f}, g[4] = {0.f, 0.f, 0.f, 0.f}, rho = 0.f;
    if (row < rows) {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(dH + row * kP) + part);
        d[0] = bf_lo(v.x), d[1] = bf_hi(v.x), d[2] = bf_lo(v.y), d[3] = bf_hi(v.y);
        const float4 a = reinterpret_cast<const float4 *>(ddH + row * kP)[part];
        g[0] = a.x, g[1] = a.y, g[2] = a.z, g[3] = a.w;
#pragma unroll
        for (int u = 0; u < 4; ++u) rho = fmaf(g[u], d[u], rho);
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) rho += __shfl_xor_sync(0xffffffffu, rho, off);
    if (row >= rows) return;
    const float rr = r[row], c3 = rr * rr * rr * rho * (1.f / kP);
    const float4 v = __ldg(reinterpret_cast<const float4 *>(gv + row * kP) + part);
    reinterpret_cast<float4 *>(ddH + row * kP)[part] =
        make_float4(v.x + rr * g[0] - c3 * d[0], v.y + rr * g[1] - c3 * d[1], v.z + rr * g[2] - c3 * d[2],
                    v.w + rr * g[3] - c3 * d[3]);
}

// Recomputation of the normalised branch. One item = a 128-token tile and a head group (the items and
// item order of the plain recompute; an order grouped by (batch row, head group), to keep the three boxes
// a chunk memory streams in L2, measured 0.15 ms slower); one step = one head and one historical chunk. Per step the tensor
// cores form U = Q Khi + Q Klo and V = C dH (N = 64 each) into one of two 128-column buffers, and the
// steps alternate between the two token warpgroups (warpgroup g takes the steps of buffer g), which share
// the head's E and dR rows and combine their halves at the end of the head.
//   pass 1 (kPass2 false): per row the online softmax statistics of its logits, (m, d) and s = sum of
//            exp(l - m) dw; at the end of a head lse (log2 units) and D = s / d into the workspace.
//   pass 2 (kPass2 true):  w, a ie and a iq ie of every (token, chunk) into the workspace, and dE.
constexpr int kNThreads = 384;  // warp 0 TMA, warp 1 MMA, warps 2-3 idle, warps 4-11 token warps
constexpr int kNStages = 2;     // a stage = one head's [Khi, Klo, dH] boxes of one chunk memory
constexpr uint32_t kN_Q = 0, kN_C = 2 * kBox, kN_H = 4 * kBox;
constexpr uint32_t kN_STG = kN_H + kNStages * 3 * kBox;  // per lane quarter 12 KiB: E rows, dR rows (2 halves)
constexpr uint32_t kN_MRG = kN_STG + 4 * 12288;          // pass 1: warpgroup 1's (m, d, s) of every row
constexpr uint32_t kN_BAR = kN_MRG + 2048;
constexpr uint32_t kN_SMEM = kN_BAR + 256 + 1024;
static_assert(kN_SMEM <= 232448, "normalised recompute kernel exceeds the shared memory of a CTA");

enum { NB_QC_FULL = 0, NB_QC_EMPTY, NB_MMA_DONE, NB_MMA_DONE2, NB_ST_FULL, NB_ST_EMPTY = NB_ST_FULL + kNStages,
       NB_UV_FULL = NB_ST_EMPTY + kNStages, NB_UV_EMPTY = NB_UV_FULL + 2, NB_LD = NB_UV_EMPTY + 2,
       NB_PAIR = NB_LD + 4, NB_COUNT = NB_PAIR + 4 };
static_assert(NB_COUNT * 8 + 8 <= 256, "barrier block overflows its 256 bytes");

struct BwdNParams {
    Shape s;
    int hpi, ngh, ntiles, multi;
    int64_t nslot, n_items;
    float eps;
    const float *iq;   // [Bt, L, G]
    float *lse2, *D;   // [Bt, H, L]: written by pass 1 (lse in log2 units), read by pass 2
    float *Wsc, *A1, *A2;  // [Bt, H, M, L]: w, a ie, a iq ie (pass 2)
    float *dE;         // [Bt, L, H, P] (pass 2)
    unsigned *amax;    // pass 2: bounds on |a ie E_t,p| and |a iq ie E_t,p| ([0], [2]) and max |dR| ([1]), float bits
};

template <bool kPass2>
__global__ void __launch_bounds__(kNThreads, 1)
    k_sma_bwd_rn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC,
                    const __grid_constant__ CUtensorMap tmKhi, const __grid_constant__ CUtensorMap tmKlo,
                    const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmE,
                    const __grid_constant__ CUtensorMap tmDR, const BwdNParams p, int *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kN_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kN_BAR + NB_COUNT * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kN_BAR + NB_COUNT * 8 + 4);
    auto bar = [&](int k) { return smem_u32(&bars[k]); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape &s = p.s;
    if (threadIdx.x == 0) {
        mbar_init(bar(NB_QC_FULL), 1);
        mbar_init(bar(NB_QC_EMPTY), 2);  // both MMA issuers commit when their MMAs of an item are done
        mbar_init(bar(NB_MMA_DONE), 1);
        mbar_init(bar(NB_MMA_DONE2), 1);
        for (int q = 0; q < kNStages; ++q) {
            mbar_init(bar(NB_ST_FULL + q), 1);
            mbar_init(bar(NB_ST_EMPTY + q), 1);
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(bar(NB_UV_FULL + q), 1);
            mbar_init(bar(NB_UV_EMPTY + q), 4);  // the four warps of the buffer's warpgroup
        }
        for (int q = 0; q < 4; ++q) {
            mbar_init(bar(NB_LD + q), 1);
            mbar_init(bar(NB_PAIR + q), 2);  // the two warps that share a lane quarter
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmKhi);
        tma_prefetch_desc(&tmKlo);
        tma_prefetch_desc(&tmH);
        tma_prefetch_desc(&tmE);
        tma_prefetch_desc(&tmDR);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        setmaxnreg_dec<kRRegsLow>();
        if (lane == 0) {
            uint32_t qc_uses = 0, ph = 0;
            int st = 0;
            int last_ph[kNStages];
            for (int q = 0; q < kNStages; ++q) last_ph[q] = -1;
            bool qc_loaded = false;
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const QItem it = q_item(s, p.ntiles, p.ngh, p.nslot, k);
                const int64_t nst = q_steps(s, it, p.multi, q_rows(s, it, p.multi));
                if (nst == 0) continue;
                const int64_t h0 = it.hg * p.hpi, grp = h0 / (s.H / s.G);
                if (!mbar_wait(bar(NB_QC_EMPTY), (qc_uses & 1) ^ 1, abort_flag, err, 151)) goto producer_end;
                mbar_arrive_expect_tx(bar(NB_QC_FULL), 4 * kBox);
                {
                    const int32_t y = (int32_t)(it.b * s.L + q_t0(s, it, p.multi));
                    for (int kh = 0; kh < 2; ++kh) {
                        tma_load_2d(sbase + kN_Q + kh * kBox, &tmQ, (int32_t)(grp * kN + kh * 64), y, bar(NB_QC_FULL));
                        tma_load_2d(sbase + kN_C + kh * kBox, &tmC, (int32_t)(grp * kN + kh * 64), y, bar(NB_QC_FULL));
                    }
                }
                ++qc_uses;
                qc_loaded = true;
                for (int hh = 0; hh < p.hpi; ++hh) {
                    for (int64_t j = 0; j < nst; ++j) {
                        if (!mbar_wait(bar(NB_ST_EMPTY + st), ph ^ 1, abort_flag, err, 152)) goto producer_end;
                        mbar_arrive_expect_tx(bar(NB_ST_FULL + st), 3 * kBox);
                        const int32_t y = (int32_t)(((it.b * s.H + h0 + hh) * s.M + j) * kN);
                        const uint32_t slot = sbase + kN_H + st * 3 * kBox;
                        tma_load_2d(slot, &tmKhi, 0, y, bar(NB_ST_FULL + st));
                        tma_load_2d(slot + kBox, &tmKlo, 0, y, bar(NB_ST_FULL + st));
                        tma_load_2d(slot + 2 * kBox, &tmH, 0, y, bar(NB_ST_FULL + st));
                        last_ph[st] = (int)ph;
                        if (++st == kNStages) {
                            st = 0;
                            ph ^= 1;
                        }
                    }
                }
            }
        producer_end:
            for (int q = 0; q < kNStages; ++q)
                if (last_ph[q] >= 0) mbar_drain(bar(NB_ST_FULL + q), (uint32_t)last_ph[q]);
            if (qc_loaded) mbar_drain(bar(NB_QC_FULL), (qc_uses - 1) & 1);
        }
    } else if (warp == 1 || warp == 2) {
        // -------------------------------- MMA ---------------------------------
        // two issuers, lane 0 of warps 1 and 2, take alternate steps (issuer i the steps of U/V buffer i)
        setmaxnreg_dec<kRRegsLow>();
        const int issuer = warp - 1;
        if (lane == 0) {
            // A = Q or C (K-major, K = N), B = one head's box (MN-major, K = N rows, N = P columns)
            constexpr uint32_t idesc = idesc_bf16_f32(kTile, kP, false, true);
            const uint64_t qdesc0 = smem_desc_sw128(sbase + kN_Q, 16, 1024);
            const uint64_t cdesc0 = smem_desc_sw128(sbase + kN_C, 16, 1024);
            uint32_t qc_uses = 0, uv = 0, ph = 0;
            int st = 0;
            bool issued = false;
            for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
                const QItem it = q_item(s, p.ntiles, p.ngh, p.nslot, k);
                const int64_t nst = q_steps(s, it, p.multi, q_rows(s, it, p.multi));
                if (nst == 0) continue;
                if (!mbar_wait(bar(NB_QC_FULL), qc_uses & 1, abort_flag, err, 161)) goto mma_end;
                ++qc_uses;
                tc_fence_after();
                for (int hh = 0; hh < p.hpi; ++hh) {
                    for (int64_t j = 0; j < nst; ++j) {
                        if ((int)(uv & 1) != issuer) {  // the other issuer's step
                            ++uv;
                            if (++st == kNStages) {
                                st = 0;
                                ph ^= 1;
                            }
                            continue;
                        }
                        if (!mbar_wait(bar(NB_ST_FULL + st), ph, abort_flag, err, 162)) goto mma_end;
                        const int ub = uv & 1;
                        if (!mbar_wait(bar(NB_UV_EMPTY + ub), ((uv >> 1) & 1) ^ 1, abort_flag, err, 163)) goto mma_end;
                        tc_fence_after();
                        const uint32_t slot = sbase + kN_H + st * 3 * kBox;
                        const uint64_t hid = smem_desc_sw128(slot, kBox, 1024);
                        const uint64_t lod = smem_desc_sw128(slot + kBox, kBox, 1024);
                        const uint64_t rwd = smem_desc_sw128(slot + 2 * kBox, kBox, 1024);
                        const uint32_t du = tmem + ub * 128, dv = du + 64;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t aoff = (uint64_t)((((kk >> 2) * kBox) + (kk & 3) * 32) >> 4);
                            const uint64_t boff = (uint64_t)((kk * 2048) >> 4);
                            mma_bf16(du, qdesc0 + aoff, hid + boff, idesc, kk > 0);
                            mma_bf16(dv, cdesc0 + aoff, rwd + boff, idesc, kk > 0);
                        }
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t aoff = (uint64_t)((((kk >> 2) * kBox) + (kk & 3) * 32) >> 4);
                            mma_bf16(du, qdesc0 + aoff, lod + (uint64_t)((kk * 2048) >> 4), idesc, 1);
                        }
                        mma_commit(bar(NB_ST_EMPTY + st));
                        mma_commit(bar(NB_UV_FULL + ub));
                        issued = true;
                        ++uv;
                        if (++st == kNStages) {
                            st = 0;
                            ph ^= 1;
                        }
                    }
                }
                mma_commit(bar(NB_QC_EMPTY));
            }
        mma_end:
            if (issued) {
                const uint32_t done = bar(issuer ? NB_MMA_DONE2 : NB_MMA_DONE);
                mma_commit(done);
                mbar_drain(done, 0);
            }
        }
    } else if (warp < 4) {
        setmaxnreg_dec<kRRegsLow>();  // no role
    } else {
        setmaxnreg_inc<kRRegsHigh>();
        // ------------------------- token warps -------------------------
        // warpgroup g takes the steps in buffer g; warp quarter = the tensor-memory lanes (token rows) it
        // owns. The two warps of a quarter share a 12 KiB staging area with the head's E and dR rows
        // (loaded by warpgroup 0's warp) and meet on a two-warp barrier at the end of every head.
        const int g = (warp - 4) >> 2, quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t stg = sbase + kN_STG + quarter * 12288;
        const uint32_t ldbar = bar(NB_LD + quarter), pairbar = bar(NB_PAIR + quarter);
        const uint32_t lrow = (uint32_t)(quarter * 32) << 16;
        const int L = (int)s.L, H = (int)s.H;
        float *mrg = reinterpret_cast<float *>(sm + kN_MRG) + row * 3;
        uint32_t tb = 0, ld_uses = 0, pair_uses = 0;
        bool ld_pending = false;
        float a1m = 0.f, a2m = 0.f, emx = 0.f, drm = 0.f;  // pass 2: maxima of |a ie|, |a iq ie|, |E|, |dR|
        for (int64_t k = blockIdx.x; k < p.n_items; k = sched_next(k)) {
            const QItem it = q_item(s, p.ntiles, p.ngh, p.nslot, k);
            const int rows = q_rows(s, it, p.multi);
            const int nsteps = (int)q_steps(s, it, p.multi, rows);
            if (nsteps == 0) continue;
            const int t0 = (int)q_t0(s, it, p.multi);
            const int t = t0 + row;
            const int b = (int)it.b;
            const bool valid = row < rows;
            const int my_chunk = valid ? (int)(t / s.S) : 0;  // the row takes the steps j < my_chunk
            const int grp = (int)(it.hg * p.hpi / (s.H / s.G));
            const float iqv = valid ? __ldg(p.iq + ((int64_t)b * L + t) * s.G + grp) : 1.f;
            for (int hh = 0; hh < p.hpi; ++hh) {
                const int h = (int)it.hg * p.hpi + hh;
                if (g == 0) {  // the head's E and dR rows into the quarter's staging area
                    __syncwarp();
                    if (lane == 0) {
                        fence_async_smem_b();
                        mbar_arrive_expect_tx(ldbar, 12288);
                        tma_load_3d(stg, &tmE, h * kP, t0 + quarter * 32, b, ldbar);
                        tma_load_3d(stg + 4096, &tmDR, h * kP, t0 + quarter * 32, b, ldbar);
                        tma_load_3d(stg + 8192, &tmDR, h * kP + 32, t0 + quarter * 32, b, ldbar);
                    }
                    ld_pending = true;
                }
                if (!mbar_wait(ldbar, ld_uses & 1, abort_flag, err, 172)) goto tok_end;
                ++ld_uses;
                ld_pending = false;
                uint32_t ev[kP / 2];  // E_t (bf16 pairs)
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    lds128(stg + lane * 128 + ((q ^ (lane & 7)) << 4), ev[4 * q], ev[4 * q + 1], ev[4 * q + 2],
                           ev[4 * q + 3]);
                float se = 0.f;
#pragma unroll
                for (int q = 0; q < kP / 2; ++q) se = fmaf(bf_lo(ev[q]), bf_lo(ev[q]), fmaf(bf_hi(ev[q]), bf_hi(ev[q]), se));
                const float iev = rsqrtf(se * (1.f / kP) + p.eps);
                const float escale = kLog2e * kRs * iqv * iev;  // l in log2 units = escale * (U' . E), U' = Q Kr
                const uint32_t dr_row = stg + 4096 + lane * 128;  // + half * 4096
                if constexpr (kPass2) {  // the fp16 row scales of the gradient GEMMs come from these maxima
#pragma unroll
                    for (int q = 0; q < kP / 2; ++q) emx = fmaxf(emx, fmaxf(fabsf(bf_lo(ev[q])), fabsf(bf_hi(ev[q]))));
                    if (g == 0) {
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            uint32_t x[4];
                            lds128(dr_row + (q >> 3) * 4096 + (((q & 7) ^ (lane & 7)) << 4), x[0], x[1], x[2], x[3]);
#pragma unroll
                            for (int w4 = 0; w4 < 4; ++w4) drm = fmaxf(drm, fabsf(__uint_as_float(x[w4])));
                        }
                    }
                }
                const int64_t hrow = (int64_t)(b * H + h) * L + t;  // [b, h, t]
                float m = -INFINITY, dsum = 0.f, ssum = 0.f;        // pass 1
                float lse2 = 0.f, Dt = 0.f;                          // pass 2
                float dEb[kP];
                if constexpr (kPass2) {
                    lse2 = valid ? p.lse2[hrow] : 0.f;
                    Dt = valid ? p.D[hrow] : 0.f;
#pragma unroll
                    for (int q = 0; q < kP; ++q) dEb[q] = 0.f;
                }
                float *wsc = p.Wsc + (int64_t)(b * H + h) * s.M * L + t;  // [b, h, j, t], j = 0
                float *a1 = p.A1 + (int64_t)(b * H + h) * s.M * L + t;
                float *a2 = p.A2 + (int64_t)(b * H + h) * s.M * L + t;
                for (int j = 0; j < nsteps; ++j) {
                    const uint32_t step = tb + (uint32_t)j;
                    if ((int)(step & 1) != g) continue;  // the other warpgroup's step
                    if (!mbar_wait(bar(NB_UV_FULL + g), (step >> 1) & 1, abort_flag, err, 173)) goto tok_end;
                    tc_fence_after();
                    const uint32_t ta = tmem + lrow + g * 128;
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int half = 0; half < 2; ++half) {  // U' . E_t
                        float u[32];
                        tmem_ld_32x32b_x32_after(ta + half * 32, u, acc[0]);
                        tmem_ld_wait_32(u);
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const uint32_t wv = ev[16 * half + q];
                            acc[q & 3] = fmaf(u[2 * q], bf_lo(wv), acc[q & 3]);
                            acc[q & 3] = fmaf(u[2 * q + 1], bf_hi(wv), acc[q & 3]);
                        }
                    }
                    const bool live = j < my_chunk;
                    const float l2 = ((acc[0] + acc[1]) + (acc[2] + acc[3])) * escale;
                    float dacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int half = 0; half < 2; ++half) {  // dw = dR_t . V (fp32 dR)
                        float v[32];
                        tmem_ld_32x32b_x32_after(ta + 64 + half * 32, v, dacc[0] + l2);
                        uint32_t dr[32];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            lds128(dr_row + half * 4096 + ((q ^ (lane & 7)) << 4), dr[4 * q], dr[4 * q + 1],
                                   dr[4 * q + 2], dr[4 * q + 3]);
                        tmem_ld_wait_32(v);
#pragma unroll
                        for (int q = 0; q < 32; ++q) dacc[q & 3] = fmaf(v[q], __uint_as_float(dr[q]), dacc[q & 3]);
                    }
                    const float dw = (dacc[0] + dacc[1]) + (dacc[2] + dacc[3]);
                    if constexpr (!kPass2) {
                        if (live) {  // online softmax statistics of the row's logits
                            if (l2 > m) {
                                const float f = exp2f(m - l2);
                                dsum *= f;
                                ssum *= f;
                                m = l2;
                            }
                            const float pw = exp2f(l2 - m);
                            dsum += pw;
                            ssum = fmaf(pw, dw, ssum);
                        }
                    } else {
                        const float w = live ? exp2f(l2 - lse2) : 0.f;
                        const float a = live ? w * (dw - Dt) * kRs : 0.f;
#pragma unroll
                        for (int half = 0; half < 2; ++half) {  // dEb += a U, U = iq U'
                            float u[32];
                            tmem_ld_32x32b_x32_after(ta + half * 32, u, a + dEb[32 * half]);
                            tmem_ld_wait_32(u);
#pragma unroll
                            for (int q = 0; q < 32; ++q) dEb[32 * half + q] = fmaf(a, u[q], dEb[32 * half + q]);
                        }
                        if (live) {
                            wsc[(int64_t)j * L] = w;
                            a1[(int64_t)j * L] = a * iev;
                            a2[(int64_t)j * L] = a * iev * iqv;
                            a1m = fmaxf(a1m, fabsf(a * iev));
                            a2m = fmaxf(a2m, fabsf(a * iev * iqv));
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(NB_UV_EMPTY + g));
                }
                tb += (uint32_t)nsteps;
                // end of the head: the two warpgroups combine their halves of every row
                if constexpr (!kPass2) {
                    if (g == 1) {
                        mrg[0] = m;
                        mrg[1] = dsum;
                        mrg[2] = ssum;
                    }
                    if (!group_sync(pairbar, pair_uses, abort_flag, err, 174)) goto tok_end;
                    if (g == 0 && valid) {
                        const float m1 = mrg[0], d1 = mrg[1], s1 = mrg[2];
                        const float mm = fmaxf(m, m1);
                        float dd = 0.f, ss = 0.f;
                        if (mm != -INFINITY) {
                            const float f0 = exp2f(m - mm), f1 = exp2f(m1 - mm);
                            dd = dsum * f0 + d1 * f1;
                            ss = ssum * f0 + s1 * f1;
                        }
                        p.lse2[hrow] = dd > 0.f ? mm + log2f(dd) : -INFINITY;
                        p.D[hrow] = dd > 0.f ? ss / dd : 0.f;
                    }
                } else {
                    // both warpgroups are done with the head's dR rows; warpgroup 1's dEb goes through them
                    if (!group_sync(pairbar, pair_uses, abort_flag, err, 175)) goto tok_end;
                    if (g == 1) {
#pragma unroll
                        for (int half = 0; half < 2; ++half)
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                sts128(dr_row + half * 4096 + ((q ^ (lane & 7)) << 4), __float_as_uint(dEb[32 * half + 4 * q]),
                                       __float_as_uint(dEb[32 * half + 4 * q + 1]), __float_as_uint(dEb[32 * half + 4 * q + 2]),
                                       __float_as_uint(dEb[32 * half + 4 * q + 3]));
                    }
                    if (!group_sync(pairbar, pair_uses, abort_flag, err, 176)) goto tok_end;
                    if (g == 0) {
                        float ed = 0.f;
#pragma unroll
                        for (int half = 0; half < 2; ++half)
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                uint32_t x[4];
                                lds128(dr_row + half * 4096 + ((q ^ (lane & 7)) << 4), x[0], x[1], x[2], x[3]);
#pragma unroll
                                for (int w4 = 0; w4 < 4; ++w4) {
                                    const int c = 32 * half + 4 * q + w4;
                                    dEb[c] = (dEb[c] + __uint_as_float(x[w4])) * iqv;  // U = iq U'
                                    ed = fmaf(c & 1 ? bf_hi(ev[c >> 1]) : bf_lo(ev[c >> 1]), dEb[c], ed);
                                }
                            }
                        if (valid) {  // dE = ie dEb - ie^3 E (E . dEb) / P
                            const float c3 = iev * iev * iev * ed * (1.f / kP);
                            float4 *de = reinterpret_cast<float4 *>(p.dE + (((int64_t)b * L + t) * H + h) * kP);
#pragma unroll
                            for (int q = 0; q < kP / 4; ++q) {
                                float o[4];
#pragma unroll
                                for (int w4 = 0; w4 < 4; ++w4) {
                                    const int c = 4 * q + w4;
                                    o[w4] = fmaf(iev, dEb[c], -c3 * (c & 1 ? bf_hi(ev[c >> 1]) : bf_lo(ev[c >> 1])));
                                }
                                de[q] = make_float4(o[0], o[1], o[2], o[3]);
                            }
                        }
                    }
                }
            }
        }
    tok_end:
        if (ld_pending) mbar_drain(ldbar, ld_uses & 1);
        if constexpr (kPass2) {  // a thread's |a ie| and |a iq ie| times its rows' largest |E| bound its products
            const float b1 = warp_max(a1m * emx), b2 = warp_max(a2m * emx), dr = warp_max(drm);
            if (p.amax && lane == 0) {
                atomicMax(p.amax, __float_as_uint(b1));
                atomicMax(p.amax + 1, __float_as_uint(dr));
                atomicMax(p.amax + 2, __float_as_uint(b2));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace

bool bwd_tc_shape_ok(const Shape &s, bool bf16) {
    const bool tiles = s.S % kTile == 0 || (s.S >= 16 && kTile % s.S == 0);  // one chunk a tile, or 128 / S
    return bf16 && s.N == kN && s.P == kP && tiles && (s.H / s.G) % 2 == 0;
}

namespace {

template <typename K>
cudaError_t prepare_tc_kernel(K kernel, int regs_expected, uint32_t smem, const char *name) {
    cudaFuncAttributes fa{};
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e == cudaSuccess && regs_expected > 0 && fa.numRegs != regs_expected) {
        set_last_error(name, cudaErrorInvalidConfiguration);
        return cudaErrorInvalidConfiguration;
    }
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) set_last_error(name, e);
    return e;
}

}  // namespace

cudaError_t launch_sma_bwd_tc(const Shape &s, const BwdArgs &a, cudaStream_t st) {
    // E per head, or e_groups = a.EG groups of hpg heads each ([Bt, L, EG, P]; the heads of a group add
    // their dE into its rows)
    const bool grouped = a.EG > 0 && a.EG != s.H;
    const int64_t EG = grouped ? a.EG : s.H;
    const int e_hpg = (int)(s.H / EG);
    // zeros where no kernel writes: dE of chunk-0 tokens (no history; all of a grouped dE, which the heads
    // add into), ddH of the last chunk memory (no later token reads it); and dQ, dC entirely, which the
    // head groups of a Q/C group add into
    const size_t S0 = (size_t)std::min(s.S, s.L);
    cudaError_t e = cudaMemsetAsync(a.dQ, 0, (size_t)(s.Bt * s.L * s.G * s.N) * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.dC, 0, (size_t)(s.Bt * s.L * s.G * s.N) * 4, st);
    if (e == cudaSuccess)
        e = grouped ? cudaMemsetAsync(a.dE, 0, (size_t)(s.Bt * s.L * EG * s.P) * 4, st)
                    : cudaMemset2DAsync(a.dE, (size_t)(s.L * s.H * s.P) * 4, 0, S0 * s.H * s.P * 4, (size_t)s.Bt, st);
    if (e == cudaSuccess)
        e = cudaMemset2DAsync(a.ddH + (s.M - 1) * s.N * s.P, (size_t)(s.M * s.N * s.P) * 4, 0,
                              (size_t)(s.N * s.P) * 4, (size_t)(s.Bt * s.H), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.amax, 0, 2 * sizeof(unsigned), st);  // maxima of |a E| and |dR|
    if (e != cudaSuccess) {
        set_last_error("cudaMemset2DAsync (gradients that take no contribution)", e);
        return e;
    }
    {
        const int64_t rows = s.Bt * s.L * s.H;
        const int64_t blocks = std::min<int64_t>((rows + 31) / 32, (int64_t)device_sm_count() * 8);
        launch_begin(KK_SMA_BWD_DELTA, st);
        k_sma_bwd_prep<<<(unsigned)blocks, 256, 0, st>>>(s, a.R, a.dR, a.D, a.amax + 1);
        if ((e = launch_end(KK_SMA_BWD_DELTA, st)) != cudaSuccess) return e;
    }
    if (s.M < 2) return cudaSuccess;  // no token has history: everything is zero
    static unsigned long long prepared = 0;  // per device
    if (!device_flag_set(prepared)) {
        if ((e = prepare_tc_kernel(k_sma_bwd_r_tc, kRRegsLaunch, kR_SMEM, "sma_bwd_r_tc setup")) != cudaSuccess ||
            (e = prepare_tc_kernel(k_sma_bwd_gq_tc<false>, 0, GqLayout<false>::kSmem, "sma_bwd_gq_tc setup")) !=
                cudaSuccess ||
            (e = prepare_tc_kernel(k_sma_bwd_gm_tc, 0, GmLayout::kSmem, "sma_bwd_gm_tc setup")) != cudaSuccess)
            return e;
        set_device_flag(&prepared);
    }
    {  // fp16 copies of dH, Q and C (16-byte vectors; N * P and G * N are multiples of 8)
        const F16Copy c0{static_cast<const uint4 *>(a.dH), static_cast<uint4 *>(a.dH16), s.Bt * s.H * s.M * s.N * s.P / 8};
        const F16Copy c1{static_cast<const uint4 *>(a.Q), static_cast<uint4 *>(a.Q16), s.Bt * s.L * s.G * s.N / 8};
        const F16Copy c2{static_cast<const uint4 *>(a.C), static_cast<uint4 *>(a.C16), s.Bt * s.L * s.G * s.N / 8};
        const int64_t blocks = std::min<int64_t>((c0.n + c1.n + c2.n + 255) / 256, (int64_t)device_sm_count() * 8);
        launch_begin(KK_SMA_BWD_F16, st);
        k_bwd_to_f16<<<(unsigned)blocks, 256, 0, st>>>(c0, c1, c2, fp16_range_word());
        if ((e = launch_end(KK_SMA_BWD_F16, st)) != cudaSuccess) return e;
    }
    const int64_t hpg = s.H / s.G;
    const int hpi = hpg % 4 == 0 ? 4 : 2;
    const int ngh = (int)(s.H / hpi);
    const bool multi = s.S < kTile;                        // 128-token tiles spanning 128 / S chunks
    const int ntiles = multi ? 1 : (int)(s.S / kTile);     // tiles per slot
    const int64_t nslots = (s.L + kTile - 1) / kTile;      // 128-token tiles of a batch row
    const int64_t nslot = multi ? nslots : s.M;            // slots of a batch row
    const int64_t n_qitems = nslot * s.Bt * ntiles * ngh;
    if (n_qitems >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
    CUtensorMap mq, mc, mh, mq16, mc16, mh16, me, mdr, mde, mdq, mdc, mddh;
    const uint64_t GN = (uint64_t)(s.G * s.N), HP = (uint64_t)(s.H * s.P), EGP = (uint64_t)(EG * s.P);
    // (the fp16 copies go through bf16 maps of the same geometry: the copy moves bytes, and no box of them
    // reaches past the tensor's end)
    if (!make_tma_map_bf16(&mq, a.Q, GN, (uint64_t)(s.Bt * s.L), GN * 2, 64, 128) ||
        !make_tma_map_bf16(&mc, a.C, GN, (uint64_t)(s.Bt * s.L), GN * 2, 64, 128) ||
        !make_tma_map_bf16(&mh, a.dH, (uint64_t)s.P, (uint64_t)(s.Bt * s.H * s.M * s.N), (uint64_t)(s.P * 2), 64, 128) ||
        !make_tma_map_bf16(&mq16, a.Q16, GN, (uint64_t)(s.Bt * s.L), GN * 2, 64, 128) ||
        !make_tma_map_bf16(&mc16, a.C16, GN, (uint64_t)(s.Bt * s.L), GN * 2, 64, 128) ||
        !make_tma_map_bf16(&mh16, a.dH16, (uint64_t)s.P, (uint64_t)(s.Bt * s.H * s.M * s.N), (uint64_t)(s.P * 2), 64,
                           128) ||
        !make_tma_map_bf16_3d(&me, a.E, EGP, (uint64_t)s.L, (uint64_t)s.Bt, EGP * 2, (uint64_t)s.L * EGP * 2, 64, 32) ||
        !make_tma_map_f32_3d(&mdr, a.dR, HP, (uint64_t)s.L, (uint64_t)s.Bt, HP * 4, (uint64_t)s.L * HP * 4, 32, 32) ||
        !make_tma_map_f32_3d(&mde, a.dE, EGP, (uint64_t)s.L, (uint64_t)s.Bt, EGP * 4, (uint64_t)s.L * EGP * 4, 32, 32) ||
        !make_tma_map_f32_3d(&mdq, a.dQ, GN, (uint64_t)s.L, (uint64_t)s.Bt, GN * 4, (uint64_t)s.L * GN * 4, 32, 32) ||
        !make_tma_map_f32_3d(&mdc, a.dC, GN, (uint64_t)s.L, (uint64_t)s.Bt, GN * 4, (uint64_t)s.L * GN * 4, 32, 32) ||
        !make_tma_map_f32_3d(&mddh, a.ddH, (uint64_t)s.P, (uint64_t)(s.Bt * s.H * s.M * s.N), 1, (uint64_t)(s.P * 4),
                             (uint64_t)(s.Bt * s.H * s.M * s.N * s.P * 4), 32, 32))
        return cudaErrorInvalidValue;
    int *err = device_error_word();
    const int64_t sms = device_sm_count();
    {
        BwdRParams p{};
        p.s = s;
        p.hpi = hpi;
        p.ngh = ngh;
        p.ntiles = ntiles;
        p.multi = multi ? 1 : 0;
        p.nslot = nslot;
        p.n_items = n_qitems;
        p.lse = a.lse;
        p.D = a.D;
        p.Wsc = a.Wsc;
        p.Asc = a.Asc;
        p.amax = a.amax;
        p.e_hpg = e_hpg;
        launch_begin(KK_SMA_BWD_R_TC, st);
        k_sma_bwd_r_tc<<<(unsigned)std::min<int64_t>(n_qitems, sms), kRThreads, kR_SMEM, st>>>(
            mq, mc, mh, me, mdr, mde, p, err);
        if ((e = launch_end(KK_SMA_BWD_R_TC, st)) != cudaSuccess) return e;
    }
    {
        BwdGParams p{};
        p.s = s;
        p.hpi = hpi;
        p.ngh = ngh;
        p.ntiles = ntiles;
        p.multi = multi ? 1 : 0;
        p.nslot = nslot;
        p.n_items = n_qitems;
        p.Wsc = a.Wsc;
        p.Asc = a.Asc;
        p.parts = 3;
        p.amax = a.amax;
        p.e_hpg = e_hpg;
        launch_begin(KK_SMA_BWD_DQ_TC, st);
        k_sma_bwd_gq_tc<false><<<(unsigned)std::min<int64_t>(n_qitems, sms), kGThreads, GqLayout<false>::kSmem, st>>>(
            mh16, mh16, me, mdr, mdq, mdc, p, err);
        if ((e = launch_end(KK_SMA_BWD_DQ_TC, st)) != cudaSuccess) return e;
    }
    {
        BwdMParams p{};
        p.s = s;
        p.nslots = nslots;
        p.nblk = (int)((s.M - 1 + kMBlock - 1) / kMBlock);
        p.n_items = (int64_t)p.nblk * s.Bt * s.H;
        p.E = static_cast<const __nv_bfloat16 *>(a.E);
        p.dR = a.dR;
        p.Wsc = a.Wsc;
        p.Asc = a.Asc;
        p.parts = 3;
        p.amax = a.amax;
        p.e_hpg = e_hpg;
        launch_begin(KK_SMA_BWD_DDH_TC, st);
        k_sma_bwd_gm_tc<<<(unsigned)std::min<int64_t>(p.n_items, sms), kGThreads, GmLayout::kSmem, st>>>(mq16, mc16, mddh,
                                                                                                      p, err);
        if ((e = launch_end(KK_SMA_BWD_DDH_TC, st)) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// ---------------------------------------------------------------------------
// Backward of the normalised score branch on the tensor cores (see k_sma_bwd_rn_tc above)
// ---------------------------------------------------------------------------

BwdNormTcWs bwd_norm_tc_layout(const Shape &s) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    BwdNormTcWs w{};
    size_t off = 0;
    const size_t bhl = (size_t)(s.Bt * s.H * s.L) * 4, pair = (size_t)(s.Bt * s.H * s.M * s.L) * 4;
    const size_t rows = (size_t)(s.Bt * s.H * s.M * s.N);
    w.D = off, off = up(off + bhl);
    w.lse2 = off, off = up(off + bhl);
    w.Wsc = off, off = up(off + pair);
    w.A1 = off, off = up(off + pair);
    w.A2 = off, off = up(off + pair);
    w.r = off, off = up(off + rows * 4);
    w.khi = off, off = up(off + rows * s.P * 2);
    w.klo = off, off = up(off + rows * s.P * 2);
    w.iq = off, off = up(off + (size_t)(s.Bt * s.L * s.G) * 4);
    w.dqb = off, off = up(off + (size_t)(s.Bt * s.L * s.G * s.N) * 4);
    w.gv = off, off = up(off + rows * s.P * 4);
    w.k16 = off, off = up(off + rows * s.P * 2);
    w.dh16 = off, off = up(off + rows * s.P * 2);
    w.q16 = off, off = up(off + (size_t)(s.Bt * s.L * s.G * s.N) * 2);
    w.c16 = off, off = up(off + (size_t)(s.Bt * s.L * s.G * s.N) * 2);
    w.amax = off, off = up(off + 256);
    w.total = off;
    return w;
}

cudaError_t launch_sma_bwd_norm_tc(const Shape &s, const BwdArgs &a, float eps, void *ws, cudaStream_t st) {
    const BwdNormTcWs wl = bwd_norm_tc_layout(s);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    float *D = reinterpret_cast<float *>(w8 + wl.D), *lse2 = reinterpret_cast<float *>(w8 + wl.lse2);
    float *W = reinterpret_cast<float *>(w8 + wl.Wsc), *A1 = reinterpret_cast<float *>(w8 + wl.A1);
    float *A2 = reinterpret_cast<float *>(w8 + wl.A2), *r = reinterpret_cast<float *>(w8 + wl.r);
    __nv_bfloat16 *khi = reinterpret_cast<__nv_bfloat16 *>(w8 + wl.khi);
    __nv_bfloat16 *klo = reinterpret_cast<__nv_bfloat16 *>(w8 + wl.klo);
    float *iq = reinterpret_cast<float *>(w8 + wl.iq), *dqb = reinterpret_cast<float *>(w8 + wl.dqb);
    float *gv = reinterpret_cast<float *>(w8 + wl.gv);
    void *k16 = w8 + wl.k16, *dh16 = w8 + wl.dh16, *q16 = w8 + wl.q16, *c16 = w8 + wl.c16;
    unsigned *amax = reinterpret_cast<unsigned *>(w8 + wl.amax);
    const size_t qbytes = (size_t)(s.Bt * s.L * s.G * s.N) * 4;
    const size_t S0 = (size_t)std::min(s.S, s.L);
    // zeros where no kernel writes or where kernels add: dC and dQb (the head groups of a Q/C group add
    // into them), dE of chunk-0 tokens, and the last chunk memory (no later token reads it) of G and GV
    cudaError_t e = cudaMemsetAsync(a.dC, 0, qbytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dqb, 0, qbytes, st);
    if (e == cudaSuccess)
        e = cudaMemset2DAsync(a.dE, (size_t)(s.L * s.H * s.P) * 4, 0, S0 * s.H * s.P * 4, (size_t)s.Bt, st);
    if (e == cudaSuccess)
        e = cudaMemset2DAsync(a.ddH + (s.M - 1) * s.N * s.P, (size_t)(s.M * s.N * s.P) * 4, 0,
                              (size_t)(s.N * s.P) * 4, (size_t)(s.Bt * s.H), st);
    if (e == cudaSuccess)
        e = cudaMemset2DAsync(gv + (s.M - 1) * s.N * s.P, (size_t)(s.M * s.N * s.P) * 4, 0, (size_t)(s.N * s.P) * 4,
                              (size_t)(s.Bt * s.H), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(amax, 0, 3 * sizeof(unsigned), st);
    if (e != cudaSuccess) {
        set_last_error("cudaMemsetAsync (normalised backward)", e);
        return e;
    }
    const int64_t rows = s.Bt * s.H * s.M * s.N, qrows = s.Bt * s.L * s.G;
    launch_begin(KK_SMA_BWD_NORM_AUX, st);
    k_norm_key_rows<<<(unsigned)((rows * 8 + 255) / 256), 256, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(a.dH), r, khi, klo, static_cast<uint4 *>(k16), static_cast<uint4 *>(dh16),
        fp16_range_word(), rows, eps);
    if ((e = launch_end(KK_SMA_BWD_NORM_AUX, st)) != cudaSuccess) return e;
    launch_begin(KK_SMA_BWD_NORM_AUX, st);
    k_norm_q_rms<<<(unsigned)((qrows * 16 + 255) / 256), 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(a.Q), iq,
                                                                       qrows, eps);
    if ((e = launch_end(KK_SMA_BWD_NORM_AUX, st)) != cudaSuccess) return e;
    if (s.M >= 2) {
        static unsigned long long prepared = 0;  // per device
        if (!device_flag_set(prepared)) {
            if ((e = prepare_tc_kernel(k_sma_bwd_rn_tc<false>, kRRegsLaunch, kN_SMEM, "sma_bwd_rn_tc setup")) !=
                    cudaSuccess ||
                (e = prepare_tc_kernel(k_sma_bwd_rn_tc<true>, kRRegsLaunch, kN_SMEM, "sma_bwd_rn_tc setup")) !=
                    cudaSuccess ||
                (e = prepare_tc_kernel(k_sma_bwd_gq_tc<true>, 0, GqLayout<true>::kSmem, "sma_bwd_gq_tc setup")) !=
                    cudaSuccess ||
                (e = prepare_tc_kernel(k_sma_bwd_gm_tc, 0, GmLayout::kSmem, "sma_bwd_gm_tc setup")) != cudaSuccess)
                return e;
            set_device_flag(&prepared);
        }
        const int64_t hpg = s.H / s.G;
        const int hpi = hpg % 4 == 0 ? 4 : 2;
        const int ngh = (int)(s.H / hpi);
        const bool multi = s.S < kTile;
        const int ntiles = multi ? 1 : (int)(s.S / kTile);
        const int64_t nslots = (s.L + kTile - 1) / kTile;
        const int64_t nslot = multi ? nslots : s.M;
        const int64_t n_qitems = nslot * s.Bt * ntiles * ngh;
        if (n_qitems >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
        CUtensorMap mq, mc, mh, mhi, mlo, mq16, mc16, mh16, mk16, me, mdr, mdqb, mdc, mddh, mgv;
        const uint64_t GN = (uint64_t)(s.G * s.N), HP = (uint64_t)(s.H * s.P);
        const uint64_t nrows = (uint64_t)(s.Bt * s.H * s.M * s.N);
        if (!make_tma_map_bf16(&mq, a.Q, GN, (uint64_t)(s.Bt * s.L), GN * 2, 64, 128) ||
            !make_tma_map_bf16(&mc, a.C, GN, (uint64_t)(s.Bt * s.L), GN * 2, 64, 128) ||
            !make_tma_map_bf16(&mh, a.dH, (uint64_t)s.P, nrows, (uint64_t)(s.P * 2), 64, 128) ||
            !make_tma_map_bf16(&mhi, khi, (uint64_t)s.P, nrows, (uint64_t)(s.P * 2), 64, 128) ||
            !make_tma_map_bf16(&mlo, klo, (uint64_t)s.P, nrows, (uint64_t)(s.P * 2), 64, 128) ||
            !make_tma_map_bf16(&mq16, q16, GN, (uint64_t)(s.Bt * s.L), GN * 2, 64, 128) ||
            !make_tma_map_bf16(&mc16, c16, GN, (uint64_t)(s.Bt * s.L), GN * 2, 64, 128) ||
            !make_tma_map_bf16(&mh16, dh16, (uint64_t)s.P, nrows, (uint64_t)(s.P * 2), 64, 128) ||
            !make_tma_map_bf16(&mk16, k16, (uint64_t)s.P, nrows, (uint64_t)(s.P * 2), 64, 128) ||
            !make_tma_map_bf16_3d(&me, a.E, HP, (uint64_t)s.L, (uint64_t)s.Bt, HP * 2, (uint64_t)s.L * HP * 2, 64, 32) ||
            !make_tma_map_f32_3d(&mdr, a.dR, HP, (uint64_t)s.L, (uint64_t)s.Bt, HP * 4, (uint64_t)s.L * HP * 4, 32, 32) ||
            !make_tma_map_f32_3d(&mdqb, dqb, GN, (uint64_t)s.L, (uint64_t)s.Bt, GN * 4, (uint64_t)s.L * GN * 4, 32, 32) ||
            !make_tma_map_f32_3d(&mdc, a.dC, GN, (uint64_t)s.L, (uint64_t)s.Bt, GN * 4, (uint64_t)s.L * GN * 4, 32, 32) ||
            !make_tma_map_f32_3d(&mddh, a.ddH, (uint64_t)s.P, nrows, 1, (uint64_t)(s.P * 4), nrows * s.P * 4, 32, 32) ||
            !make_tma_map_f32_3d(&mgv, gv, (uint64_t)s.P, nrows, 1, (uint64_t)(s.P * 4), nrows * s.P * 4, 32, 32))
            return cudaErrorInvalidValue;
        int *err = device_error_word();
        const int64_t sms = device_sm_count();
        const unsigned qgrid = (unsigned)std::min<int64_t>(n_qitems, sms);
        {  // fp16 copies of Q and C for the gradient GEMMs (those of dH and the key rows came with r)
            const F16Copy c0{nullptr, nullptr, 0};
            const F16Copy c1{static_cast<const uint4 *>(a.Q), static_cast<uint4 *>(q16), s.Bt * s.L * s.G * s.N / 8};
            const F16Copy c2{static_cast<const uint4 *>(a.C), static_cast<uint4 *>(c16), s.Bt * s.L * s.G * s.N / 8};
            const int64_t blocks = std::min<int64_t>((c1.n + c2.n + 255) / 256, sms * 8);
            launch_begin(KK_SMA_BWD_F16, st);
            k_bwd_to_f16<<<(unsigned)blocks, 256, 0, st>>>(c0, c1, c2, fp16_range_word());
            if ((e = launch_end(KK_SMA_BWD_F16, st)) != cudaSuccess) return e;
        }
        BwdNParams np{};
        np.s = s;
        np.hpi = hpi;
        np.ngh = ngh;
        np.ntiles = ntiles;
        np.multi = multi ? 1 : 0;
        np.nslot = nslot;
        np.n_items = n_qitems;
        np.eps = eps;
        np.iq = iq;
        np.lse2 = lse2;
        np.D = D;
        np.Wsc = W;
        np.A1 = A1;
        np.A2 = A2;
        np.dE = a.dE;
        np.amax = amax;
        launch_begin(KK_SMA_BWD_RN_TC, st);
        k_sma_bwd_rn_tc<false><<<qgrid, kNThreads, kN_SMEM, st>>>(mq, mc, mhi, mlo, mh, me, mdr, np, err);
        if ((e = launch_end(KK_SMA_BWD_RN_TC, st)) != cudaSuccess) return e;
        launch_begin(KK_SMA_BWD_RN_TC, st);
        k_sma_bwd_rn_tc<true><<<qgrid, kNThreads, kN_SMEM, st>>>(mq, mc, mhi, mlo, mh, me, mdr, np, err);
        if ((e = launch_end(KK_SMA_BWD_RN_TC, st)) != cudaSuccess) return e;
        BwdGParams gp{};
        gp.s = s;
        gp.hpi = hpi;
        gp.ngh = ngh;
        gp.ntiles = ntiles;
        gp.multi = multi ? 1 : 0;
        gp.nslot = nslot;
        gp.n_items = n_qitems;
        gp.Wsc = W;
        gp.Asc = A1;
        gp.amax = amax;  // [0] bounds the rows a ie E, [1] the rows w dR
        // dC = sum w dH dR against the memories; dQb = sum (a ie E) Kr^T against the key rows (fp16 both)
        gp.parts = 3;
        launch_begin(KK_SMA_BWD_DQ_TC, st);
        k_sma_bwd_gq_tc<true><<<qgrid, kGThreads, GqLayout<true>::kSmem, st>>>(mh16, mk16, me, mdr, mdqb, mdc, gp, err);
        if ((e = launch_end(KK_SMA_BWD_DQ_TC, st)) != cudaSuccess) return e;
        BwdMParams mp{};
        mp.s = s;
        mp.nslots = nslots;
        mp.nblk = (int)((s.M - 1 + kMBlock - 1) / kMBlock);
        mp.n_items = (int64_t)mp.nblk * s.Bt * s.H;
        mp.E = static_cast<const __nv_bfloat16 *>(a.E);
        mp.dR = a.dR;
        mp.Wsc = W;
        mp.Asc = A2;
        mp.amax = amax;
        mp.key_amax = 2;  // the rows a iq ie E
        // G = sum Q^T (a iq ie E) into ddH, then GV = sum C^T (w dR) into the workspace (fp16, each with its
        // own row scale)
        const unsigned mgrid = (unsigned)std::min<int64_t>(mp.n_items, sms);
        mp.parts = 1;
        launch_begin(KK_SMA_BWD_DDH_TC, st);
        k_sma_bwd_gm_tc<<<mgrid, kGThreads, GmLayout::kSmem, st>>>(mq16, mc16, mddh, mp, err);
        if ((e = launch_end(KK_SMA_BWD_DDH_TC, st)) != cudaSuccess) return e;
        mp.parts = 2;
        launch_begin(KK_SMA_BWD_DDH_TC, st);
        k_sma_bwd_gm_tc<<<mgrid, kGThreads, GmLayout::kSmem, st>>>(mq16, mc16, mgv, mp, err);
        if ((e = launch_end(KK_SMA_BWD_DDH_TC, st)) != cudaSuccess) return e;
    } else {  // no token has history: dQb, G and GV stay zero
        const size_t mem = (size_t)rows * s.P * 4;
        e = cudaMemsetAsync(a.ddH, 0, mem, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(gv, 0, mem, st);
        if (e != cudaSuccess) {
            set_last_error("cudaMemsetAsync (normalised backward)", e);
            return e;
        }
    }
    launch_begin(KK_SMA_BWD_NORM_AUX, st);
    k_norm_dq_post<<<(unsigned)((qrows * 16 + 255) / 256), 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(a.Q), iq,
                                                                         dqb, a.dQ, qrows);
    if ((e = launch_end(KK_SMA_BWD_NORM_AUX, st)) != cudaSuccess) return e;
    launch_begin(KK_SMA_BWD_NORM_AUX, st);
    k_norm_ddh_combine<<<(unsigned)((rows * 16 + 255) / 256), 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(a.dH),
                                                                            r, gv, a.ddH, rows);
    return launch_end(KK_SMA_BWD_NORM_AUX, st);
}

}  // namespace dart
