// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dart.h"

namespace dart {

// Kernel kinds, for launch counting and per-kernel timing.
enum KernelKind : int {
    KK_CHUNK_CUMSUM = 0,   // a1: within-chunk log-decay cumsum and chunk totals
    KK_CHUNK_STATES = 1,   // a2: dH[c] (CUDA cores)
    KK_CHUNK_STATES_TC,    // a2: dH[c] (tcgen05)
    KK_STATE_PASS,         // a3: chunk-boundary scan (warp shuffles)
    KK_SSD_OUT,            // a4: Y (CUDA cores)
    KK_SSD_OUT_TC,         // a4: Y (tcgen05)
    KK_SMA_FWD,            // a5/a6: SMA (+ combine) (CUDA cores)
    KK_SMA_FWD_TC,         // a5/a6: SMA (+ combine) (tcgen05)
    KK_SMA_DECODE,         // a7: decode partials over cached chunks
    KK_DECODE_MERGE,       // a7: merge of decode partials + combine
    KK_DECODE_STATE,       // decode step: recurrent state, open chunk memory, cache append
    KK_SMA_FWD_NORM_TC,    // SMA with the normalised score branch (tcgen05)
    KK_SMA_BWD_DELTA,      // SMA backward: D_t = dR_t . R_t
    KK_SMA_BWD_DQ,         // SMA backward, query side: dQ, dC, dE (CUDA cores)
    KK_SMA_BWD_DDH,        // SMA backward, memory side: d dH (CUDA cores)
    KK_SMA_BWD_R_TC,       // SMA backward, recomputation: dE and the chunk weights (tcgen05)
    KK_SMA_BWD_DQ_TC,      // SMA backward, dQ and dC GEMMs (tcgen05)
    KK_SMA_BWD_DDH_TC,     // SMA backward, ddH GEMMs (tcgen05)
    KK_KEY_RMS,            // normalised branch: fp16 key rows r (.) dH and fp16 Q rows, prepared once
    KK_SMA_BWD_RN_TC,      // normalised-branch backward: recomputed statistics, weights and dE (tcgen05)
    KK_SMA_BWD_NORM_AUX,   // normalised-branch backward: key rows, RMS factors, dQ and ddH assembly
    KK_SMA_BWD_F16,        // SMA backward: fp16 copies of dH, Q and C for the gradient GEMMs
    KK_COUNT
};

const char *kernel_name(int kind);

// Records the reason of the last failure for dart_last_error().
void set_last_error(const char *where, cudaError_t e);

// Launch bookkeeping: every kernel launch goes through these two calls.
void launch_begin(int kind, cudaStream_t stream);
cudaError_t launch_end(int kind, cudaStream_t stream);

struct Shape {
    int64_t Bt, L, H, G, N, P, S, M;
};

// Device pointers of one layer call (unused ones are null).
struct LayerPtrs {
    const void *X, *B, *C, *Q, *E;
    const float *logA;
    const float *g;
    int64_t g_sb, g_st, g_sh;
    float *cs;       // [Bt, H, L] within-chunk inclusive cumsum of logA (workspace)
    float *lam;      // [Bt, H, M] chunk totals (workspace)
    void *dH;        // [Bt, H, M, N, P]
    void *Hprev;     // [Bt, H, M, N, P] state entering each chunk (workspace)
    float *final_state;
    void *Y;         // fp32 SSD output (or `out` for the fused layer)
    void *R;         // fp32 SMA readout (sma_fwd only)
    float *lse;
    bool combine;    // fused layer: the SMA epilogue adds g R into out, which holds the SSD output Y
    bool score_norm;  // SMA with the normalised score branch (App. B.1 eq 25-27), epsilon norm_eps
    float norm_eps;
    int64_t e_groups;  // E [Bt, L, e_groups, P], head h reading group h / (H / e_groups); 0 = one per head
    void *norm_prep;   // normalised branch, tensor cores: scratch for the prepared operands (norm_prep_layout), or
                       // null: the SMA kernel rescales the key rows and the Q tile itself
};

// heads per E group (1 when E is per head)
__host__ __device__ inline int64_t heads_per_e(const Shape &s, int64_t e_groups) { return e_groups > 0 ? s.H / e_groups : 1; }

// ---- CUDA-core kernels (any supported shape; fp32 or bf16 storage) ----
cudaError_t launch_chunk_cumsum(const Shape &s, const float *logA, float *cs, float *lam, cudaStream_t st);
cudaError_t launch_chunk_states_simt(const Shape &s, bool bf16, const LayerPtrs &p, cudaStream_t st);
cudaError_t launch_state_pass(const Shape &s, bool bf16, const LayerPtrs &p, cudaStream_t st);
cudaError_t launch_ssd_out_simt(const Shape &s, bool bf16, const LayerPtrs &p, cudaStream_t st);
cudaError_t launch_sma_fwd_simt(const Shape &s, bool bf16, const LayerPtrs &p, cudaStream_t st);

// SMA backward (gradients of R by recomputation with the forward's lse)
struct BwdArgs {
    const void *Q, *C, *E, *dH;  // forward inputs, in the input dtype
    const float *R, *lse, *dR;   // forward readout and logsumexp; dLoss/dR
    float *D;                    // [Bt, H, L] workspace: D_t = dR_t . R_t
    float *dQ, *dC, *dE, *ddH;   // gradients, fp32, layouts of Q, C, E and dH
    // tensor-core path only (workspace): w and a = dl / sqrt(N) per (token, chunk, head)
    float *Wsc, *Asc;            // [Bt, H, M, L]
    // tensor-core path only (workspace): dH, Q and C as fp16 for the gradient GEMMs, and two maxima as the
    // bits of non-negative floats: [0] of |a E_t| over every (token, chunk, head), [1] of |dR|
    void *dH16, *Q16, *C16;
    unsigned *amax;
    // normalised-branch backward only (workspace): the recomputed lse, [Bt, H, L]; lse points here too
    float *lse_rc;
    // grouped E (CUDA-core kernels): E and dE are [Bt, L, EG, P], head h reading group h / (H / EG);
    // EG = 0 or H: one per head. With fewer groups dE is zeroed first and the heads add into it.
    int64_t EG;
};

// E row of (token row bt, head h) in a [Bt, L, EG, P] layout
__host__ __device__ inline int64_t e_row(const Shape &s, int64_t EG, int64_t bt, int64_t h) {
    return (EG > 0 && EG != s.H) ? bt * EG + h / (s.H / EG) : bt * s.H + h;
}

// tensor-core backward: bf16, N = 128, P = 64, S % 128 == 0, H / G even
bool bwd_tc_shape_ok(const Shape &s, bool bf16);

cudaError_t launch_sma_bwd_delta(const Shape &s, const BwdArgs &a, cudaStream_t st);
cudaError_t launch_sma_bwd_simt(const Shape &s, bool bf16, const BwdArgs &a, cudaStream_t st);
cudaError_t launch_sma_bwd_norm_simt(const Shape &s, bool bf16, const BwdArgs &a, float eps, cudaStream_t st);
cudaError_t launch_sma_bwd_tc(const Shape &s, const BwdArgs &a, cudaStream_t st);
// Backward of the normalised score branch on the tensor cores (the shapes of bwd_tc_shape_ok); its scratch
struct BwdNormTcWs {
    size_t D, lse2, Wsc, A1, A2, r, khi, klo, iq, dqb, gv, k16, dh16, q16, c16, amax, total;
};
BwdNormTcWs bwd_norm_tc_layout(const Shape &s);
cudaError_t launch_sma_bwd_norm_tc(const Shape &s, const BwdArgs &a, float eps, void *ws, cudaStream_t st);

struct DecodeArgs {
    int64_t Bt, H, G, N, P, n_chunks, chunk_stride;
    const void *Q, *C, *E, *Y;
    const float *g;
    int64_t g_sb, g_sh;
    const void *cache;
    void *out;
    float *lse;
    float *partials;  // [Bt, H, splits, 2 + P]
    int splits;
    bool y_f32;       // Y is fp32 (the decode step's own Y) rather than in the input dtype
    int64_t EG;       // E [Bt, EG, P], head h reading group h / (H / EG); 0 = one per head
};

// One decode step's state maintenance (the recurrence of eq (2) for one token): state and the open
// chunk's memory take a B^T X, Y = C state; on a chunk close the memory goes to cache slot n_chunks.
struct StateStepArgs {
    int64_t Bt, H, G, N, P, n_chunks, chunk_stride;
    int close_chunk;
    const void *X, *B, *C;
    const float *logA;
    float *state, *acc;
    void *cache;
    float *Y;  // [Bt, H, P] fp32
};
cudaError_t launch_decode_state(const StateStepArgs &a, bool bf16, cudaStream_t st);
int decode_splits(int64_t Bt, int64_t H, int64_t n_chunks);
cudaError_t launch_sma_decode(const DecodeArgs &a, bool bf16, cudaStream_t st);

// ---- host helpers of the tcgen05 kernels ----
// 2D bf16 TMA map over a row-major [rows, cols] matrix (`row_bytes` apart), box
// box_cols x box_rows, 128-byte swizzle, zero fill out of bounds. `map` points to
// a CUtensorMap. Records the reason in dart_last_error on failure.
bool make_tma_map_bf16(void *map, const void *base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                       uint32_t box_cols, uint32_t box_rows);
// bf16 3-D tiled map (d0 innermost, 128-byte swizzle), boxes of box0 x box1 x 1: rows (d1) that run
// past the end of a batch row read as zeros instead of the next batch row.
bool make_tma_map_bf16_3d(void *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
                          uint64_t stride2_bytes, uint32_t box0, uint32_t box1);
// fp32 3-D tiled map (d0 innermost, 128-byte swizzle), boxes of box0 x box1 x 1; used for stores
// whose rows must clip at the end of every batch row (d1) rather than run into the next.
bool make_tma_map_f32_3d(void *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
                         uint64_t stride2_bytes, uint32_t box0, uint32_t box1);
int device_sm_count();
// Per-device one-time kernel setup: whether the current device's bit is set in a flag word (one bit per
// device; devices 64 and up always read as not set), and setting it once the setup has succeeded.
bool device_flag_set(unsigned long long flags);
void set_device_flag(unsigned long long *flags);

// ---- tcgen05 kernels (bf16, N = 128, P = 64, S % 128 == 0) ----
bool tc_shape_ok(const Shape &s, bool bf16);
// tensor-core SMA with a grouped E (any number of heads per group)
inline bool tc_shape_ok_ge(const Shape &s, bool bf16, int64_t e_groups) {
    (void)e_groups;  // any grouping: the kernel reads E group h / (H / e_groups)
    return tc_shape_ok(s, bf16);
}
cudaError_t launch_sma_fwd_tc(const Shape &s, const LayerPtrs &p, cudaStream_t st);
// scratch of the normalised branch's prepared operands: the key rows r (.) dH in fp16 [Bt, H, M, N, P], the
// Q rows scaled to fp16 [Bt, L, G, N] and their remaining factors [Bt, L, G] fp32 (byte offsets)
struct NormPrepWs {
    size_t k16, q16, qfac, total;
};
NormPrepWs norm_prep_layout(const Shape &s);
bool states_tc_shape_ok(const Shape &s, bool bf16);  // also needs S in {128, 256}
cudaError_t launch_chunk_states_tc(const Shape &s, const LayerPtrs &p, int *err_word, cudaStream_t st);
bool ssd_tc_shape_ok(const Shape &s, bool bf16);  // also needs S in {128, 256}
cudaError_t launch_ssd_out_tc(const Shape &s, const LayerPtrs &p, int *err_word, cudaStream_t st);
// device address of the error word the tcgen05 kernels write (per device, cached)
int *device_error_word();

// Device error word written by kernels that gave up a bounded wait (0 = none).
int read_device_error(bool clear);
// Wait limit of the bounded waits of the tensor-core kernels on the current device (nanoseconds).
cudaError_t set_wait_limit_ns(unsigned long long ns);

// Range flags of the tensor-core kernels that multiply fp16 operands: a kernel ORs in its bit when it
// wrote a non-finite value (an fp16 operand overflowed, or an input was not finite).
enum { kRangeChunkStates = 1, kRangeSsdOut = 2, kRangeBwdOperands = 4 };
int *fp16_range_word();  // per device, cached; null when the lookup failed
int read_fp16_range(bool clear);

// ---- small device helpers ----
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

}  // namespace dart
