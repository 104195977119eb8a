/*
 * dart.h -- C ABI of the DART forward hot path on NVIDIA B200 (sm_100a).
 *
 * DART ("Decoded Attention over Recurrent States for Efficient Long-Context
 * Sequence Modeling", arXiv 2608.02032) keeps the chunk state contributions of
 * the Mamba-2 chunked SSD scan as chunk state memories dH[c] and attends over
 * them with token-conditioned keys and values (state-memory attention, SMA).
 * This library computes, on one GPU:
 *
 *   chunk state memories  dH[c] = sum_{s in c} A_{s+1:e(c)} B_s^T X_s           (§3 eq 5)
 *   SSD scan output       Y_t = C_t H_t, H_t = a_t H_{t-1} + B_t^T X_t          (§2 eq 2, App. A eq 17-24)
 *   state-memory attention for c < chunk(t):
 *                         V = C_t dH[c], K = dH[c] E_t, l = Q_t K / sqrt(N)     (§3 eq 8-9)
 *                         R_t = sum_c softmax_c(l) V,  lse_t = logsumexp_c(l)   (§3 eq 10; Alg. 1)
 *   gated residual        out_t = Y_t + g_t R_t                                 (§3 eq 11)
 *   single-token decode   SMA of one new token over every cached dH[c]          (§4 "Inference Cache")
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Indexing: tokens and chunks are 0-based, chunk(t) = t / S, M = ceil(L / S).
 *   The last chunk may be short (L % S != 0). Tokens of chunk 0 have no history:
 *   R_t = 0 and lse_t = -inf there (§3, text after eq 10; Alg. 1 steps 15-16).
 * Decay: logA_t = log a_t is given per (batch, token, head) in fp32; a_t multiplies
 *   the previous state only, so a token's own write is undecayed at that token
 *   (eq 2, with A_{u:v} = I for u > v, eq 3).
 * Layouts (row-major, contiguous, element strides implied by the shape):
 *   X, E             [batch, L, H, P]        in `dtype`
 *   Y, R, out        [batch, L, H, P]        fp32
 *   B, C, Q          [batch, L, G, N]        in `dtype`; head h reads group h / (H / G)
 *   logA             [batch, L, H]           fp32
 *   dH               [batch, H, M, N, P]     in `dtype`
 *   lse              [batch, H, L]           fp32
 *   final_state      [batch, H, N, P]        fp32
 *   g                fp32, element (b, t, h) at g[b*g_sb + t*g_st + h*g_sh]; a stride of 0 broadcasts
 * Memory: every pointer is caller-owned DEVICE memory, 16-byte aligned; the
 *   library never allocates or frees device memory. Scratch is passed as `ws`
 *   (256-byte aligned) of at least dart_workspace_size() / dart_decode_workspace_size()
 *   bytes; its contents on entry do not matter and are clobbered.
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *   stream). Calls only enqueue work and never synchronise; outputs are ready
 *   when the stream reaches them. The device current at call time is used.
 * Arithmetic: bf16 inputs are multiplied on tensor cores (or CUDA cores) with
 *   fp32 accumulation; softmax, decays and the recurrence run in fp32. The
 *   chunk memories dH (the decode cache) are stored in `dtype`; Y, R, out and
 *   lse are stored in fp32, because the SSD output is heavy-tailed (max/rms
 *   near 10) and a bf16 rounding of it alone would cost up to 4% of its rms.
 *   fp32 inputs use fp32 FMA throughout (no TF32).
 * fp16 range of the tensor-core scan: with bf16 inputs, N = 128 and P = 64 the
 *   chunk-state and SSD-output kernels multiply some operands in fp16, which
 *   keeps 11 significant bits but ends at 65504: in dart_chunk_states the rows B_s
 *   and the decay-scaled rows exp(sum_{r=s+1}^{e(c)} logA_r) X_s; in the SSD
 *   output (dart_ssd_scan, dart_layer_fwd) the rows X_s and the intra-chunk
 *   weights (C_t . B_s) exp(sum_{r=s+1}^{t} logA_r), s <= t in one chunk. With
 *   logA <= 0 the limits are |B|, |X| < 65504 and |C_t . B_s| < 65504. An operand
 *   past the limit becomes inf (one in [65504, 65520) rounds to 65504), so the
 *   outputs it reaches are written as inf or NaN, never as a wrong finite value,
 *   and the kernel raises its bit in dart_fp16_range_flags(). An overflowed X_s
 *   reaches the chunk memory of its chunk and head, and the SSD output of every
 *   token of its 128-token block (the products run over whole blocks, 0 * inf
 *   included) and of the later chunks of that head. The CUDA-core kernels (fp32
 *   inputs, other shapes) have no such limit.
 * Errors: arguments are checked on the host before anything is enqueued; on a
 *   bad argument the call returns a non-zero dart_status and leaves every output
 *   untouched. A failed kernel launch returns DART_ERR_CUDA (cudaGetLastError
 *   is consumed). No entry point traps or aborts.
 */
#ifndef DART_H
#define DART_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DART_OK = 0,
    DART_ERR_NULL = 1,        /* a required pointer is NULL */
    DART_ERR_DIMS = 2,        /* a size is <= 0, or H % G != 0, or sizes overflow */
    DART_ERR_DTYPE = 3,       /* unknown dart_dtype */
    DART_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned (workspace: 256-byte) */
    DART_ERR_UNSUPPORTED = 5, /* shape outside what the kernels handle (see dart_supported) */
    DART_ERR_WORKSPACE = 6,   /* ws is NULL or ws_bytes is smaller than required */
    DART_ERR_CUDA = 7         /* a CUDA launch or runtime call failed */
} dart_status;

typedef enum { DART_F32 = 0, DART_BF16 = 1 } dart_dtype;

typedef enum {
    DART_OP_CHUNK_STATES = 0,
    DART_OP_SSD_SCAN = 1,
    DART_OP_SMA_FWD = 2,
    DART_OP_LAYER_FWD = 3,
    DART_OP_SMA_BWD = 4,
    DART_OP_SMA_BWD_NORM = 5,
    DART_OP_SMA_FWD_NORM = 6
} dart_op;

/* Problem sizes. batch, seqlen L, nheads H, ngroups G (B, C, Q shared by H/G heads),
 * dstate N (state/key size), headdim P (value size), chunk S. */
typedef struct {
    int64_t batch, seqlen, nheads, ngroups, dstate, headdim, chunk;
} dart_dims;

/* Human-readable name of a status code (static storage). */
const char *dart_status_string(dart_status status);

/* Library version string (static storage). */
const char *dart_version(void);

/* DART_OK when the kernels handle these sizes: 1 <= N <= 256, 1 <= P <= 256,
 * N * P <= 16384, 1 <= S <= 1024, H % G == 0. bf16 with N = 128, P = 64 runs the
 * tensor-core (tcgen05) kernels: the chunk memories for S in {16, 32, 64, 128, 256},
 * the scan and SSD output for S in {128, 256} (and, for S < 128, on 256-token chunks
 * of their own, see dart_ssd_scan), the SMA forward and both backward branches for S
 * a multiple of 128 or a divisor of 128 (S >= 16) with H / G even. Every other
 * supported shape runs fp32 CUDA-core kernels. */
dart_status dart_supported(const dart_dims *dims, dart_dtype dtype);

/* Bytes of `ws` the op needs for these sizes (0 when none). Sizes that are not
 * supported return 0; the op itself then reports the error. */
size_t dart_workspace_size(dart_op op, const dart_dims *dims, dart_dtype dtype);

/* Chunk state memories, eq (5):  dH[c] = sum_{s in c} exp(sum_{r=s+1}^{e(c)} logA_r) B_s^T X_s.
 * In: X, B, logA. Out: dH [batch, H, M, N, P]. Scratch: ws (DART_OP_CHUNK_STATES). */
dart_status dart_chunk_states(const dart_dims *dims, dart_dtype dtype, const void *X, const void *B,
                              const float *logA, void *dH, void *ws, size_t ws_bytes, void *stream);

/* SSD scan output from chunk state memories (App. A eq 17-24): state passing
 * H_[c] = exp(sum_{r in c} logA_r) H_[c-1] + dH[c] (eq 18), then
 * Y_t = sum_{s in c, s <= t} (C_t . B_s) A_{s+1:t} X_s + C_t A_{a_c:t} H_[c-1]  (eq 21-22).
 * In: X, B, C, logA, dH (as written by dart_chunk_states). Out: Y; final_state
 * (fp32 H after the last token) when not NULL. Scratch: ws (DART_OP_SSD_SCAN).
 * The result is the recurrence of eq (2) whatever the chunking: for bf16, N = 128,
 * P = 64 and S < 128 the scan runs on 256-token chunks whose memories it forms
 * itself from X, B, logA in the workspace, and dH is not read. */
dart_status dart_ssd_scan(const dart_dims *dims, dart_dtype dtype, const void *X, const void *B, const void *C,
                          const float *logA, const void *dH, void *Y, float *final_state, void *ws, size_t ws_bytes,
                          void *stream);

/* State-memory attention forward (eq 8-10; Algorithm 1): for every token t with
 * chunk(t) >= 1, attention over dH[0 .. chunk(t)-1] with keys dH[c] E_t, values
 * C_t dH[c] and logits Q_t K / sqrt(N). In: Q, C, E, dH. Out: R; lse when not NULL.
 * Tokens of chunk 0 get R = 0 and lse = -inf. No scratch. */
dart_status dart_sma_fwd(const dart_dims *dims, dart_dtype dtype, const void *Q, const void *C, const void *E,
                         const void *dH, void *R, float *lse, void *stream);

/* Grouped E (the MVA-style grouped projections of the Fig. 2 caption and App. B.2,
 * where B, C, Q and E share one projection group, G = 1): E is [batch, L, e_groups, P]
 * and head h reads E group h / (H / e_groups). 1 <= e_groups <= H with H % e_groups == 0,
 * else DART_ERR_DIMS; e_groups = H is the per-head layout of dart_sma_fwd, which calls
 * this with e_groups = H. Every other argument, output and rule as dart_sma_fwd. */
dart_status dart_sma_fwd_ge(const dart_dims *dims, dart_dtype dtype, int64_t e_groups, const void *Q, const void *C,
                            const void *E, const void *dH, void *R, float *lse, void *stream);

/* State-memory attention with the normalised score branch of App. B.1 (the
 * "in practice" form of §3, eq 25-27):
 *   Qb_t = Q_t / sqrt(mean_n Q_t^2 + eps),  Eb_t = E_t / sqrt(mean_p E_t^2 + eps)   (eq 25)
 *   r_{c,n} = (mean_p dH[c]_{n,p}^2 + eps)^(-1/2),  K = r_c (.) (dH[c] Eb_t)         (eq 26)
 *   l = Qb_t K / sqrt(N), softmax over c < chunk(t), R_t = sum_c g_c C_t dH[c]      (eq 27)
 * RMSNorm has unit weight; the value side C_t dH[c] is not normalised.
 * Arguments, layouts and outputs as dart_sma_fwd; eps >= 0 (finite), else
 * DART_ERR_DIMS. dH is read only. bf16 with N = 128, P = 64 runs on the tensor
 * cores, the key product in fp16 (rescaled key rows rounded once to fp16); other
 * shapes and fp32 run on the CUDA-core kernel in fp32. No scratch. */
dart_status dart_sma_fwd_norm(const dart_dims *dims, dart_dtype dtype, const void *Q, const void *C, const void *E,
                              const void *dH, void *R, float *lse, float eps, void *stream);

/* dart_sma_fwd_norm with scratch ws of dart_workspace_size(DART_OP_SMA_FWD_NORM)
 * bytes (0 for shapes off the tensor-core path; ws may then be NULL): on the tensor
 * cores a pass before the SMA kernel writes into ws the key rows r_c (.) dH[c] rounded
 * once to fp16 ([batch, H, M, N, P]), the Q rows scaled by the power of two at or
 * below their RMSNorm factor to fp16 ([batch, L, G, N]) and the rest of that factor
 * ([batch, L, G] fp32), and the SMA kernel reads them instead of rescaling every
 * staged row itself. ws = NULL with ws_bytes = 0 is dart_sma_fwd_norm; a non-NULL ws
 * smaller than the size, or misaligned, is DART_ERR_WORKSPACE. Results as
 * dart_sma_fwd_norm (the same fp16 operands; r's sum of squares may add in another
 * order). */
dart_status dart_sma_fwd_norm_ws(const dart_dims *dims, dart_dtype dtype, const void *Q, const void *C,
                                 const void *E, const void *dH, void *R, float *lse, float eps, void *ws,
                                 size_t ws_bytes, void *stream);

/* State-memory attention backward by recomputation (§4 "Efficient Training": the
 * forward stores only R and lse; chunk keys, values, logits and weights are
 * recomputed; App. C eq 32-35 recovers the weights as w_c = exp(l_c - lse_t)).
 * For a loss with gradient dR = dLoss/dR, per token t (chunk(t) >= 1) and head h:
 *   dw_c = dR_t . (C_t dH[c]),  D_t = dR_t . R_t,  dl_c = w_c (dw_c - D_t),
 *   dQ_t += dl_c (dH[c] E_t) / sqrt(N),     dC_t += w_c dH[c] dR_t,
 *   dE_t += dl_c dH[c]^T Q_t / sqrt(N),     ddH[c] += w_c C_t^T dR_t + dl_c Q_t^T E_t / sqrt(N).
 * dQ and dC sum over the heads of a group; lse takes no gradient.
 * In: Q, C, E, dH (the forward's inputs, dtype), R and lse as dart_sma_fwd wrote
 * them (fp32), dR (fp32, layout of R). Out (fp32, every element written):
 * dQ, dC [batch, L, G, N], dE [batch, L, H, P], ddH [batch, H, M, N, P]; tokens of
 * chunk 0 and chunk memories no later token reads get exact zeros.
 * Scratch: ws of dart_workspace_size(DART_OP_SMA_BWD) bytes (D, batch * H * L
 * floats; on the tensor cores also w and dl / sqrt(N) of every (token, chunk, head)
 * and fp16 copies of dH, Q and C). bf16 with N = 128, P = 64 runs on the tensor
 * cores: keys, values and weights recomputed in bf16 x bf16 products with fp32
 * accumulation, the gradient products in fp16 (dH, Q and C converted, exact for
 * magnitudes up to 65280; the rows dl_c E_t and w_c dR_t rounded once after a
 * power-of-two scale that keeps the largest of them below 2^14, removed again in
 * fp32). A dH, Q or C value of 65536 or more becomes inf there, so the gradients it
 * reaches are not finite, and raises bit 2 of dart_fp16_range_flags(). Every other
 * shape runs on CUDA cores in fp32. */
dart_status dart_sma_bwd(const dart_dims *dims, dart_dtype dtype, const void *Q, const void *C, const void *E,
                         const void *dH, const float *R, const float *lse, const float *dR, float *dQ, float *dC,
                         float *dE, float *ddH, void *ws, size_t ws_bytes, void *stream);

/* dart_sma_bwd with a grouped E, [batch, L, e_groups, P] (see dart_sma_fwd_ge): head h
 * reads E group h / (H / e_groups), and dE ([batch, L, e_groups, P], fp32) is the sum over
 * the heads of each group of their per-head gradients. e_groups = H is dart_sma_bwd,
 * which calls this. For e_groups < H dE is zeroed and every head adds its gradient into
 * its group's rows (a TMA reduce-add on the tensor-core shapes of dart_sma_bwd, atomic
 * adds on the CUDA-core kernels), so the rounding order of dE may vary from call to call;
 * the engine and scratch are those of dart_sma_bwd for the same sizes. 1 <= e_groups <= H
 * with H % e_groups == 0, else DART_ERR_DIMS. */
dart_status dart_sma_bwd_ge(const dart_dims *dims, dart_dtype dtype, int64_t e_groups, const void *Q, const void *C,
                            const void *E, const void *dH, const float *R, const float *lse, const float *dR,
                            float *dQ, float *dC, float *dE, float *ddH, void *ws, size_t ws_bytes, void *stream);

/* Backward of the normalised score branch (dart_sma_fwd_norm; App. B.1 eq 25-27), by
 * recomputation as dart_sma_bwd: R and lse are those dart_sma_fwd_norm wrote, eps the
 * same. With a_c = w_c (dR_t . V_c - dR_t . R_t) / sqrt(N):
 *   dQb = sum_c a_c K_c, dEb = sum_c a_c dH[c]^T (r_c (.) Qb), dC as dart_sma_bwd,
 *   ddH[c]_{n,p} += w_c C_n dR_p + a_c Qb_n (r_n Eb_p - r_n^3 (dH[c] Eb)_n dH[c]_{n,p} / P),
 *   dQ_t = iq dQb - iq^3 Q_t (Q_t . dQb) / N, dE_t = ie dEb - ie^3 E_t (E_t . dEb) / P
 * (iq, ie: the RMSNorm factors of Q_t and E_t). Outputs, layouts and zeros as
 * dart_sma_bwd. The softmax statistics (lse and D_t = sum_c w_c dw_c) are recomputed
 * from the logits, so R and lse are not read and may be NULL (they keep the signature
 * of dart_sma_bwd; the tensor-core forward's fp16 keys make its lse too coarse for
 * gradients). Scratch: ws (DART_OP_SMA_BWD_NORM). bf16 with N = 128, P = 64 and the
 * chunk sizes of the tensor-core dart_sma_bwd runs on the tensor cores: the key rows
 * r_c (.) dH[c] enter as bf16 hi + lo pairs (16 significant bits, for the logits and
 * dQ), everything else as dart_sma_bwd; fp32 accumulation. Every other shape runs on
 * CUDA cores in fp32. */
dart_status dart_sma_bwd_norm(const dart_dims *dims, dart_dtype dtype, float eps, const void *Q, const void *C,
                              const void *E, const void *dH, const float *R, const float *lse, const float *dR,
                              float *dQ, float *dC, float *dE, float *ddH, void *ws, size_t ws_bytes, void *stream);

/* The whole DART mixer forward: chunk states -> state passing -> SSD output Y
 * (written into `out`) -> SMA, whose epilogue adds g R into `out` (the gated
 * residual out = Y + g R, eq 11), so R never goes through HBM.
 * In: X, B, C, Q, E, logA, g (+ strides). Out: out; dH_out (the chunk memory
 * cache for decode); lse_out when not NULL. With g = 0 everywhere, out equals
 * the Y of dart_ssd_scan bit for bit. Scratch: ws (DART_OP_LAYER_FWD). */
dart_status dart_layer_fwd(const dart_dims *dims, dart_dtype dtype, const void *X, const void *B, const void *C,
                           const void *Q, const void *E, const float *logA, const float *g, int64_t g_sb,
                           int64_t g_st, int64_t g_sh, void *out, void *dH_out, float *lse_out, void *ws,
                           size_t ws_bytes, void *stream);

/* dart_layer_fwd with a grouped E, [batch, L, e_groups, P] (see dart_sma_fwd_ge); dart_layer_fwd
 * calls this with e_groups = H. */
dart_status dart_layer_fwd_ge(const dart_dims *dims, dart_dtype dtype, int64_t e_groups, const void *X, const void *B,
                              const void *C, const void *Q, const void *E, const float *logA, const float *g,
                              int64_t g_sb, int64_t g_st, int64_t g_sh, void *out, void *dH_out, float *lse_out,
                              void *ws, size_t ws_bytes, void *stream);

/* Bytes of scratch dart_sma_decode needs (0 for unsupported sizes). */
size_t dart_decode_workspace_size(int64_t batch, int64_t nheads, int64_t dstate, int64_t headdim, int64_t n_chunks,
                                  dart_dtype dtype);

/* Single-token SMA decode (§4 "Inference Cache"): one new token per batch row
 * attends over the n_chunks completed chunk memories in the cache (all of them
 * are historical), then out = Y + g R.
 * In:  Q, C [batch, G, N]; E, Y [batch, H, P] (all in `dtype`); g fp32 at
 *      g[b*g_sb + h*g_sh]; cache [batch, H, chunk_stride, N, P] in `dtype` with
 *      chunk_stride >= n_chunks (capacity).
 * Out: out [batch, H, P] fp32; lse [batch, H] fp32 when not NULL.
 * n_chunks = 0 gives out = Y and lse = -inf. Scratch: ws. */
dart_status dart_sma_decode(int64_t batch, int64_t nheads, int64_t ngroups, int64_t dstate, int64_t headdim,
                            int64_t n_chunks, int64_t chunk_stride, dart_dtype dtype, const void *Q, const void *C,
                            const void *E, const void *Y, const float *g, int64_t g_sb, int64_t g_sh,
                            const void *cache, void *out, float *lse, void *ws, size_t ws_bytes, void *stream);

/* dart_sma_decode with a grouped E, [batch, e_groups, P] (see dart_sma_fwd_ge); dart_sma_decode
 * calls this with e_groups = nheads. */
dart_status dart_sma_decode_ge(int64_t batch, int64_t nheads, int64_t ngroups, int64_t e_groups, int64_t dstate,
                               int64_t headdim, int64_t n_chunks, int64_t chunk_stride, dart_dtype dtype,
                               const void *Q, const void *C, const void *E, const void *Y, const float *g,
                               int64_t g_sb, int64_t g_sh, const void *cache, void *out, float *lse, void *ws,
                               size_t ws_bytes, void *stream);

/* Bytes of scratch dart_decode_step needs (0 for unsupported sizes). */
size_t dart_decode_step_workspace_size(int64_t batch, int64_t nheads, int64_t dstate, int64_t headdim,
                                       int64_t n_chunks, dart_dtype dtype);

/* One decode step of the whole mixer, with the state it keeps between steps
 * (§4 "Inference Cache": the recurrent state and the chunk memories are what a
 * decoder caches; §2 eq (2) in recurrent form; §3 eq (5) accumulated token by
 * token). For one new token per batch row, with a = exp(logA):
 *   state     <- a * state + B^T X                  (the full state H_t, eq 2)
 *   chunk_acc <- a * chunk_acc + B^T X              (the memory of the open chunk)
 *   Y         =  C state                            (eq 2)
 *   out       =  Y + g R                            (eq 11), R = the SMA readout of the
 *                token over the n_chunks cached memories (eq 8-10, as dart_sma_decode)
 * and, when close_chunk is nonzero (the token is the last of its chunk), the
 * call stores chunk_acc, rounded to `dtype`, as cache slot n_chunks and resets
 * chunk_acc to zero; the next token's call then passes n_chunks + 1. The token
 * never reads its own chunk's memory (the readout uses slots < n_chunks).
 * Stepping a sequence this way gives the out, lse, chunk memories and final
 * state of the parallel forward (dart_layer_fwd) for every token.
 * In:  X, E [batch, H, P]; B, C, Q [batch, G, N] (all in `dtype`); logA [batch, H]
 *      fp32 (the token's log decay); g fp32 at g[b*g_sb + h*g_sh].
 * In/out: state, chunk_acc [batch, H, N, P] fp32 (zero before the first token);
 *      cache [batch, H, chunk_stride, N, P] in `dtype`, slots [0, n_chunks) filled.
 * Out: out [batch, H, P] fp32; lse [batch, H] fp32 when not NULL.
 * Errors: DART_ERR_DIMS also when close_chunk is set and n_chunks == chunk_stride
 * (no free slot); nothing is launched then. Scratch: ws
 * (dart_decode_step_workspace_size). Shapes as dart_sma_decode. */
dart_status dart_decode_step(int64_t batch, int64_t nheads, int64_t ngroups, int64_t dstate, int64_t headdim,
                             int64_t n_chunks, int64_t chunk_stride, int close_chunk, dart_dtype dtype,
                             const void *X, const void *B, const void *C, const void *Q, const void *E,
                             const float *logA, const float *g, int64_t g_sb, int64_t g_sh, float *state,
                             float *chunk_acc, void *cache, void *out, float *lse, void *ws, size_t ws_bytes,
                             void *stream);

/* dart_sma_decode without a workspace argument, for callers that cannot allocate
 * device memory: code handed only its input and output buffers by a framework
 * that owns every allocation (a plug-in inside a serving system, say, whose
 * request threads may not call cudaMalloc because it can synchronise the device
 * and can fail under memory pressure). The paper has no counterpart: this is a
 * deployment convenience of this library.
 * Arguments, layouts and results are those of dart_sma_decode. The split
 * partials go to a fixed 4 MiB device array inside the library instead of `ws`;
 * every GPU that loads the library holds that array until the process exits.
 * Sizes whose partials exceed it (batch * nheads * splits * (2 + headdim) * 4
 * bytes, the size dart_decode_workspace_size reports) return DART_ERR_WORKSPACE
 * without launching anything. The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current and
 * keeps it; make that first call before any stream capture, and do not use this
 * entry point on a device again after cudaDeviceReset has torn down its context
 * (the kept address would be stale). The call allocates nothing. All
 * calls on a device share the array: nothing in it needs to start at zero (each
 * call writes every partial it reads), but calls whose kernels overlap on the
 * GPU race on it and must be serialised by the caller. */
dart_status dart_sma_decode_noalloc(int64_t batch, int64_t nheads, int64_t ngroups, int64_t dstate,
                                    int64_t headdim, int64_t n_chunks, int64_t chunk_stride, dart_dtype dtype,
                                    const void *Q, const void *C, const void *E, const void *Y, const float *g,
                                    int64_t g_sb, int64_t g_sh, const void *cache, void *out, float *lse,
                                    void *stream);

/* ---- introspection (host side only) ------------------------------------ */

/* Device error word of the current device, then cleared: 0 when no kernel has
 * given up since the last read; otherwise the code of the first wait that ran
 * out (every wait inside the tensor-core kernels is bounded, by default to 2 s,
 * see dart_set_wait_limit; on expiry the kernel stops, lets its copies and tensor
 * core products in flight finish, releases its tensor memory and returns, leaving
 * its outputs incomplete). Synchronises the device; -1 if the read itself failed. */
int dart_device_error(void);

/* Wait limit of the tensor-core kernels on the current device, in nanoseconds:
 * a kernel whose bounded wait makes no progress for this long stops as
 * dart_device_error describes. ns = 0 restores the default of 2 s; more than
 * 10 s is DART_ERR_DIMS. A short limit makes the kernels give up on purpose (a
 * test of that path); kernels already enqueued may see either value. The waits
 * with which a stopping kernel lets its own copies and products finish always
 * allow 2 s. Synchronous (cudaMemcpyToSymbol). */
dart_status dart_set_wait_limit(uint64_t ns);

/* fp16 range flags of the current device, then cleared: bit 0 (1) when the
 * tensor-core chunk-state kernel wrote a chunk memory that is not finite, bit 1
 * (2) when the tensor-core SSD-output kernel wrote a non-finite output, bit 2 (4)
 * when the tensor-core SMA backward met a dH, Q or C value that fp16 cannot hold
 * (see dart_sma_bwd), since the last read. With finite inputs a raised bit means
 * that an fp16 operand overflowed (see "fp16 range" above); a non-finite input
 * raises it too. 0 when none happened. Synchronises the device; -1 if the read
 * itself failed. */
int dart_fp16_range_flags(void);

/* Text of the last CUDA failure behind a DART_ERR_CUDA status (which call, the
 * CUDA error name and message); empty when none happened. Static storage. */
const char *dart_last_error(void);

/* Kernels this library has launched in this process so far. */
int64_t dart_kernel_launches(void);

/* Number of kernel kinds and the name of kind `id` (NULL when out of range). */
int dart_kernel_kinds(void);
const char *dart_kernel_name(int id);

/* Per-kernel device timing: while enabled, every launch is bracketed by CUDA
 * events recorded on its stream. dart_profile_read waits for the recorded
 * events, returns the summed milliseconds and launch count of kernel kind `id`
 * since the last reset, and keeps the records; dart_profile_reset drops them. */
dart_status dart_profile_enable(int enable);
dart_status dart_profile_read(int id, double *total_ms, int64_t *launches);
dart_status dart_profile_reset(void);

#ifdef __cplusplus
}
#endif

#endif /* DART_H */
