// C ABI entry points of the DART forward path: argument checks, workspace
// carving, kernel dispatch, launch counting and optional per-kernel timing.
#include <atomic>
#include <cstdio>
#include <cmath>
#include <mutex>
#include <vector>

#include "dart_internal.cuh"

namespace dart {

const char *last_error();

// ---------------------------------------------------------------------------
// launch bookkeeping
// ---------------------------------------------------------------------------

static const char *kKernelNames[KK_COUNT] = {
    "chunk_cumsum",  "chunk_states", "chunk_states_tc", "state_pass", "ssd_out",
    "ssd_out_tc",    "sma_fwd",      "sma_fwd_tc",      "sma_decode", "decode_merge",
    "decode_state",  "sma_fwd_norm_tc", "sma_bwd_delta", "sma_bwd_dq", "sma_bwd_ddh",
    "sma_bwd_r_tc",  "sma_bwd_dq_tc",   "sma_bwd_ddh_tc", "sma_norm_prep", "sma_bwd_rn_tc", "sma_bwd_norm_aux",
    "sma_bwd_f16",
};

const char *kernel_name(int kind) { return (kind >= 0 && kind < KK_COUNT) ? kKernelNames[kind] : nullptr; }

namespace {
std::atomic<int64_t> g_launches{0};
std::mutex g_mu;
bool g_profile = false;
struct Rec {
    cudaEvent_t a, b;
};
std::vector<Rec> g_recs[KK_COUNT];
cudaEvent_t g_open[KK_COUNT];
bool g_has_open[KK_COUNT];

cudaEvent_t new_event() {
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}
}  // namespace

void launch_begin(int kind, cudaStream_t stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_profile) return;
    cudaEvent_t e = new_event();
    cudaEventRecord(e, stream);
    g_open[kind] = e;
    g_has_open[kind] = true;
}

namespace {
std::mutex g_err_mu;
char g_last_error[512] = "";
}  // namespace

void set_last_error(const char *where, cudaError_t e) {
    std::lock_guard<std::mutex> lk(g_err_mu);
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

const char *last_error() {
    std::lock_guard<std::mutex> lk(g_err_mu);
    return g_last_error;
}

cudaError_t launch_end(int kind, cudaStream_t stream) {
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
    else set_last_error(kernel_name(kind), err);
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_profile && g_has_open[kind]) {
        cudaEvent_t e = new_event();
        cudaEventRecord(e, stream);
        g_recs[kind].push_back({g_open[kind], e});
        g_has_open[kind] = false;
    }
    return err;
}

}  // namespace dart

using namespace dart;

namespace {

constexpr int64_t kMaxGrid = 65535;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

dart_status check_dims(const dart_dims *d, Shape *s) {
    if (!d) return DART_ERR_NULL;
    if (d->batch <= 0 || d->seqlen <= 0 || d->nheads <= 0 || d->ngroups <= 0 || d->dstate <= 0 || d->headdim <= 0 ||
        d->chunk <= 0)
        return DART_ERR_DIMS;
    if (d->nheads % d->ngroups != 0) return DART_ERR_DIMS;
    if (d->batch > kMaxGrid || d->nheads > kMaxGrid || d->seqlen > (int64_t(1) << 40)) return DART_ERR_DIMS;
    s->Bt = d->batch;
    s->L = d->seqlen;
    s->H = d->nheads;
    s->G = d->ngroups;
    s->N = d->dstate;
    s->P = d->headdim;
    s->S = d->chunk;
    s->M = (d->seqlen + d->chunk - 1) / d->chunk;
    return DART_OK;
}

dart_status check_supported(const Shape &s, dart_dtype dt) {
    if (dt != DART_F32 && dt != DART_BF16) return DART_ERR_DTYPE;
    if (s.N > 256 || s.P > 256 || s.N * s.P > 16384 || s.S > 1024) return DART_ERR_UNSUPPORTED;
    if (s.M * ((s.S + 15) / 16) > (int64_t(1) << 31) - 1) return DART_ERR_UNSUPPORTED;
    return DART_OK;
}

size_t esize(dart_dtype dt) { return dt == DART_BF16 ? 2 : 4; }

struct WsLayout {
    size_t cs, lam, hprev, total;
};

// SMA backward scratch: D [Bt, H, L]; on the tensor-core path also the per-pair scalars w and
// dl / sqrt(N) [Bt, H, M, L] each, fp16 copies of dH [Bt, H, M, N, P] and of Q and C [Bt, L, G, N],
// and two maxima (256 bytes)
struct BwdWs {
    size_t D, Wsc, Asc, dH16, Q16, C16, amax, total;
};

BwdWs bwd_layout(const Shape &s, bool tc) {
    BwdWs w{};
    size_t off = 0;
    w.D = off;
    off = round_up(off + (size_t)(s.Bt * s.H * s.L) * sizeof(float), 256);
    if (tc) {
        w.Wsc = off;
        off = round_up(off + (size_t)(s.Bt * s.H * s.M * s.L) * sizeof(float), 256);
        w.Asc = off;
        off = round_up(off + (size_t)(s.Bt * s.H * s.M * s.L) * sizeof(float), 256);
        w.dH16 = off;
        off = round_up(off + (size_t)(s.Bt * s.H * s.M * s.N * s.P) * 2, 256);
        w.Q16 = off;
        off = round_up(off + (size_t)(s.Bt * s.L * s.G * s.N) * 2, 256);
        w.C16 = off;
        off = round_up(off + (size_t)(s.Bt * s.L * s.G * s.N) * 2, 256);
        w.amax = off;
        off += 256;
    }
    w.total = off;
    return w;
}

size_t bwd_ws(const Shape &s, dart_dtype dt) { return bwd_layout(s, bwd_tc_shape_ok(s, dt == DART_BF16)).total; }

// normalised-branch forward scratch (tensor-core shapes): r of every chunk memory row, [Bt, H, M, N]
size_t sma_norm_ws(const Shape &s, dart_dtype dt) {
    return tc_shape_ok(s, dt == DART_BF16) ? norm_prep_layout(s).total : 0;
}

// normalised-branch backward scratch: on the tensor cores the layout of bwd_norm_tc_layout; on CUDA
// cores D and the recomputed lse, [Bt, H, L] each
size_t bwd_norm_ws(const Shape &s, dart_dtype dt) {
    if (bwd_tc_shape_ok(s, dt == DART_BF16)) return bwd_norm_tc_layout(s).total;
    return 2 * round_up((size_t)(s.Bt * s.H * s.L) * sizeof(float), 256);
}

WsLayout layer_ws(const Shape &s, dart_dtype dt, bool need_hprev) {
    WsLayout w{};
    size_t off = 0;
    w.cs = off;
    off = round_up(off + (size_t)(s.Bt * s.H * s.L) * sizeof(float), 256);
    w.lam = off;
    off = round_up(off + (size_t)(s.Bt * s.H * s.M) * sizeof(float), 256);
    w.hprev = off;
    if (need_hprev) off = round_up(off + (size_t)(s.Bt * s.H * s.M * s.N * s.P) * esize(dt), 256);
    w.total = off;
    return w;
}

// The SSD output and the scan are the recurrence of eq (2) whatever the chunking: for a chunk size the
// tensor-core scan does not take (S < 128) the scan runs on 256-token chunks of its own, with their own
// cumsum, chunk memories (workspace) and state passing; only the SMA and its memories use S.
Shape scan256_shape(const Shape &s) {
    Shape r = s;
    r.S = 256;
    r.M = (s.L + 255) / 256;
    return r;
}

bool use_scan256(const Shape &s, bool bf16) {
    const Shape r = scan256_shape(s);
    return s.S < 128 && ssd_tc_shape_ok(r, bf16) && states_tc_shape_ok(r, bf16);
}

struct Scan256Ws {
    size_t cs, lam, dH, hprev, end;
};

Scan256Ws scan256_ws(const Shape &s, dart_dtype dt, size_t off) {
    const Shape r = scan256_shape(s);
    Scan256Ws w{};
    w.cs = off;
    off = round_up(off + (size_t)(r.Bt * r.H * r.L) * sizeof(float), 256);
    w.lam = off;
    off = round_up(off + (size_t)(r.Bt * r.H * r.M) * sizeof(float), 256);
    w.dH = off;
    off = round_up(off + (size_t)(r.Bt * r.H * r.M * r.N * r.P) * esize(dt), 256);
    w.hprev = off;
    off = round_up(off + (size_t)(r.Bt * r.H * r.M * r.N * r.P) * esize(dt), 256);
    w.end = off;
    return w;
}

// scratch of the layer and of the scan
size_t layer_ws_bytes(const Shape &s, dart_dtype dt) {
    if (use_scan256(s, dt == DART_BF16)) return scan256_ws(s, dt, layer_ws(s, dt, false).total).end;
    return layer_ws(s, dt, true).total;
}

size_t scan_ws_bytes(const Shape &s, dart_dtype dt) {
    if (use_scan256(s, dt == DART_BF16)) return scan256_ws(s, dt, 0).end;
    return layer_ws(s, dt, true).total;
}

dart_status check_ws(void *ws, size_t ws_bytes, size_t need) {
    if (need == 0) return DART_OK;
    if (!ws || ws_bytes < need) return DART_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return DART_ERR_ALIGN;
    return DART_OK;
}

#define DART_TRY_PTR(p)                         \
    do {                                        \
        if (!(p)) return DART_ERR_NULL;         \
        if (!aligned((p), 16)) return DART_ERR_ALIGN; \
    } while (0)
#define DART_OPT_PTR(p)                                 \
    do {                                                \
        if ((p) && !aligned((p), 16)) return DART_ERR_ALIGN; \
    } while (0)

dart_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DART_OK : DART_ERR_CUDA; }

// Chunk states: tensor cores for the bf16 N=128 P=64 S in {128, 256} shapes, CUDA cores otherwise.
cudaError_t launch_chunk_states(const Shape &s, bool bf16, const LayerPtrs &p, cudaStream_t st) {
    if (states_tc_shape_ok(s, bf16)) return launch_chunk_states_tc(s, p, device_error_word(), st);
    return launch_chunk_states_simt(s, bf16, p, st);
}

// SSD output: tensor cores for the bf16 N=128 P=64 S in {128, 256} shapes, CUDA cores otherwise.
cudaError_t launch_ssd_out(const Shape &s, bool bf16, const LayerPtrs &p, cudaStream_t st) {
    if (ssd_tc_shape_ok(s, bf16)) return launch_ssd_out_tc(s, p, device_error_word(), st);
    return launch_ssd_out_simt(s, bf16, p, st);
}

// The scan and SSD output on 256-token chunks (see use_scan256); `p` carries X, B, C, logA and Y (written
// here; in the fused layer the SMA epilogue adds g R to it afterwards); base is the workspace.
cudaError_t launch_scan256(const Shape &s, bool bf16, LayerPtrs p, char *base, const Scan256Ws &w,
                           cudaStream_t st) {
    const Shape r = scan256_shape(s);
    p.cs = reinterpret_cast<float *>(base + w.cs);
    p.lam = reinterpret_cast<float *>(base + w.lam);
    p.dH = base + w.dH;
    p.Hprev = base + w.hprev;
    cudaError_t e = launch_chunk_cumsum(r, p.logA, p.cs, p.lam, st);
    if (e == cudaSuccess) e = launch_chunk_states(r, bf16, p, st);
    if (e == cudaSuccess) e = launch_state_pass(r, bf16, p, st);
    if (e == cudaSuccess) e = launch_ssd_out(r, bf16, p, st);
    return e;
}

#define DART_LAUNCH(expr)                         \
    do {                                          \
        cudaError_t _e = (expr);                  \
        if (_e != cudaSuccess) return DART_ERR_CUDA; \
    } while (0)

}  // namespace

extern "C" {

const char *dart_status_string(dart_status status) {
    switch (status) {
        case DART_OK: return "ok";
        case DART_ERR_NULL: return "a required pointer is NULL";
        case DART_ERR_DIMS: return "invalid sizes";
        case DART_ERR_DTYPE: return "unknown dtype";
        case DART_ERR_ALIGN: return "misaligned pointer";
        case DART_ERR_UNSUPPORTED: return "unsupported shape";
        case DART_ERR_WORKSPACE: return "workspace missing or too small";
        case DART_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

const char *dart_version(void) { return "dart-b200 0.1.0 (sm_100a)"; }

dart_status dart_supported(const dart_dims *dims, dart_dtype dtype) {
    Shape s;
    dart_status st = check_dims(dims, &s);
    if (st != DART_OK) return st;
    return check_supported(s, dtype);
}

size_t dart_workspace_size(dart_op op, const dart_dims *dims, dart_dtype dtype) {
    Shape s;
    if (check_dims(dims, &s) != DART_OK || check_supported(s, dtype) != DART_OK) return 0;
    switch (op) {
        case DART_OP_CHUNK_STATES: return layer_ws(s, dtype, false).total;
        case DART_OP_SSD_SCAN: return scan_ws_bytes(s, dtype);
        case DART_OP_SMA_FWD: return 0;
        case DART_OP_LAYER_FWD: return layer_ws_bytes(s, dtype);
        case DART_OP_SMA_BWD: return bwd_ws(s, dtype);
        case DART_OP_SMA_BWD_NORM: return bwd_norm_ws(s, dtype);
        case DART_OP_SMA_FWD_NORM: return sma_norm_ws(s, dtype);
    }
    return 0;
}

dart_status dart_chunk_states(const dart_dims *dims, dart_dtype dtype, const void *X, const void *B,
                              const float *logA, void *dH, void *ws, size_t ws_bytes, void *stream) {
    Shape s;
    dart_status st = check_dims(dims, &s);
    if (st != DART_OK) return st;
    if ((st = check_supported(s, dtype)) != DART_OK) return st;
    DART_TRY_PTR(X);
    DART_TRY_PTR(B);
    DART_TRY_PTR(logA);
    DART_TRY_PTR(dH);
    WsLayout w = layer_ws(s, dtype, false);
    if ((st = check_ws(ws, ws_bytes, w.total)) != DART_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == DART_BF16;
    LayerPtrs p{};
    p.X = X;
    p.B = B;
    p.logA = logA;
    p.dH = dH;
    p.cs = reinterpret_cast<float *>(static_cast<char *>(ws) + w.cs);
    p.lam = reinterpret_cast<float *>(static_cast<char *>(ws) + w.lam);
    DART_LAUNCH(launch_chunk_cumsum(s, logA, p.cs, p.lam, cs));
    DART_LAUNCH(launch_chunk_states(s, bf16, p, cs));
    return DART_OK;
}

dart_status dart_ssd_scan(const dart_dims *dims, dart_dtype dtype, const void *X, const void *B, const void *C,
                          const float *logA, const void *dH, void *Y, float *final_state, void *ws, size_t ws_bytes,
                          void *stream) {
    Shape s;
    dart_status st = check_dims(dims, &s);
    if (st != DART_OK) return st;
    if ((st = check_supported(s, dtype)) != DART_OK) return st;
    DART_TRY_PTR(X);
    DART_TRY_PTR(B);
    DART_TRY_PTR(C);
    DART_TRY_PTR(logA);
    DART_TRY_PTR(dH);
    DART_TRY_PTR(Y);
    DART_OPT_PTR(final_state);
    if ((st = check_ws(ws, ws_bytes, scan_ws_bytes(s, dtype))) != DART_OK) return st;
    WsLayout w = layer_ws(s, dtype, true);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == DART_BF16;
    LayerPtrs p{};
    p.X = X;
    p.B = B;
    p.C = C;
    p.logA = logA;
    p.dH = const_cast<void *>(dH);
    p.Y = Y;
    p.final_state = final_state;
    if (use_scan256(s, bf16)) {  // the same recurrence on 256-token chunks (dH of the S-token chunks unused)
        DART_LAUNCH(launch_scan256(s, bf16, p, static_cast<char *>(ws), scan256_ws(s, dtype, 0), cs));
        return DART_OK;
    }
    p.cs = reinterpret_cast<float *>(static_cast<char *>(ws) + w.cs);
    p.lam = reinterpret_cast<float *>(static_cast<char *>(ws) + w.lam);
    p.Hprev = static_cast<char *>(ws) + w.hprev;
    DART_LAUNCH(launch_chunk_cumsum(s, logA, p.cs, p.lam, cs));
    DART_LAUNCH(launch_state_pass(s, bf16, p, cs));
    DART_LAUNCH(launch_ssd_out(s, bf16, p, cs));
    return DART_OK;
}

static bool e_groups_ok(const Shape &s, int64_t e_groups) {
    return e_groups >= 1 && e_groups <= s.H && s.H % e_groups == 0;
}

dart_status dart_sma_fwd(const dart_dims *dims, dart_dtype dtype, const void *Q, const void *C, const void *E,
                         const void *dH, void *R, float *lse, void *stream) {
    return dart_sma_fwd_ge(dims, dtype, dims ? dims->nheads : 0, Q, C, E, dH, R, lse, stream);
}

dart_status dart_sma_fwd_ge(const dart_dims *dims, dart_dtype dtype, int64_t e_groups, const void *Q, const void *C,
                            const void *E, const void *dH, void *R, float *lse, void *stream) {
    Shape s;
    dart_status st = check_dims(dims, &s);
    if (st != DART_OK) return st;
    if ((st = check_supported(s, dtype)) != DART_OK) return st;
    if (!e_groups_ok(s, e_groups)) return DART_ERR_DIMS;
    DART_TRY_PTR(Q);
    DART_TRY_PTR(C);
    DART_TRY_PTR(E);
    DART_TRY_PTR(dH);
    DART_TRY_PTR(R);
    DART_OPT_PTR(lse);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == DART_BF16;
    LayerPtrs p{};
    p.Q = Q;
    p.C = C;
    p.E = E;
    p.dH = const_cast<void *>(dH);
    p.R = R;
    p.lse = lse;
    p.combine = false;
    p.e_groups = e_groups;
    if (tc_shape_ok_ge(s, bf16, e_groups)) {
        DART_LAUNCH(launch_sma_fwd_tc(s, p, cs));
    } else {
        DART_LAUNCH(launch_sma_fwd_simt(s, bf16, p, cs));
    }
    return DART_OK;
}

dart_status dart_sma_fwd_norm(const dart_dims *dims, dart_dtype dtype, const void *Q, const void *C, const void *E,
                              const void *dH, void *R, float *lse, float eps, void *stream) {
    return dart_sma_fwd_norm_ws(dims, dtype, Q, C, E, dH, R, lse, eps, nullptr, 0, stream);
}

dart_status dart_sma_fwd_norm_ws(const dart_dims *dims, dart_dtype dtype, const void *Q, const void *C,
                                 const void *E, const void *dH, void *R, float *lse, float eps, void *ws,
                                 size_t ws_bytes, void *stream) {
    Shape s;
    dart_status st = check_dims(dims, &s);
    if (st != DART_OK) return st;
    if ((st = check_supported(s, dtype)) != DART_OK) return st;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return DART_ERR_DIMS;
    // no scratch: the tensor-core kernel rescales the staged key rows and the Q tile itself
    const size_t need = sma_norm_ws(s, dtype);
    if (ws || ws_bytes) {
        if ((st = check_ws(ws, ws_bytes, need)) != DART_OK) return st;
    }
    DART_TRY_PTR(Q);
    DART_TRY_PTR(C);
    DART_TRY_PTR(E);
    DART_TRY_PTR(dH);
    DART_TRY_PTR(R);
    DART_OPT_PTR(lse);
    LayerPtrs p{};
    p.Q = Q;
    p.C = C;
    p.E = E;
    p.dH = const_cast<void *>(dH);
    p.R = R;
    p.lse = lse;
    p.combine = false;
    p.score_norm = true;
    p.norm_eps = eps;
    p.norm_prep = (ws && need) ? ws : nullptr;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (tc_shape_ok(s, dtype == DART_BF16)) {
        DART_LAUNCH(launch_sma_fwd_tc(s, p, cs));
    } else {
        DART_LAUNCH(launch_sma_fwd_simt(s, dtype == DART_BF16, p, cs));
    }
    return DART_OK;
}

dart_status dart_sma_bwd(const dart_dims *dims, dart_dtype dtype, const void *Q, const void *C, const void *E,
                         const void *dH, const float *R, const float *lse, const float *dR, float *dQ, float *dC,
                         float *dE, float *ddH, void *ws, size_t ws_bytes, void *stream) {
    return dart_sma_bwd_ge(dims, dtype, dims ? dims->nheads : 0, Q, C, E, dH, R, lse, dR, dQ, dC, dE, ddH, ws,
                           ws_bytes, stream);
}

dart_status dart_sma_bwd_ge(const dart_dims *dims, dart_dtype dtype, int64_t e_groups, const void *Q, const void *C,
                            const void *E, const void *dH, const float *R, const float *lse, const float *dR,
                            float *dQ, float *dC, float *dE, float *ddH, void *ws, size_t ws_bytes, void *stream) {
    Shape s;
    dart_status st = check_dims(dims, &s);
    if (st != DART_OK) return st;
    if ((st = check_supported(s, dtype)) != DART_OK) return st;
    if (!e_groups_ok(s, e_groups)) return DART_ERR_DIMS;
    DART_TRY_PTR(Q);
    DART_TRY_PTR(C);
    DART_TRY_PTR(E);
    DART_TRY_PTR(dH);
    DART_TRY_PTR(R);
    DART_TRY_PTR(lse);
    DART_TRY_PTR(dR);
    DART_TRY_PTR(dQ);
    DART_TRY_PTR(dC);
    DART_TRY_PTR(dE);
    DART_TRY_PTR(ddH);
    const bool grouped = e_groups != s.H;
    const bool tc = bwd_tc_shape_ok(s, dtype == DART_BF16);
    const BwdWs wl = bwd_layout(s, tc);
    if ((st = check_ws(ws, ws_bytes, wl.total)) != DART_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    BwdArgs a{};
    a.Q = Q;
    a.C = C;
    a.E = E;
    a.dH = dH;
    a.R = R;
    a.lse = lse;
    a.dR = dR;
    a.D = static_cast<float *>(ws);
    a.dQ = dQ;
    a.dC = dC;
    a.dE = dE;
    a.ddH = ddH;
    a.EG = grouped ? e_groups : 0;
    if (tc) {
        uint8_t *w8 = static_cast<uint8_t *>(ws);
        a.D = reinterpret_cast<float *>(w8 + wl.D);
        a.Wsc = reinterpret_cast<float *>(w8 + wl.Wsc);
        a.Asc = reinterpret_cast<float *>(w8 + wl.Asc);
        a.dH16 = w8 + wl.dH16;
        a.Q16 = w8 + wl.Q16;
        a.C16 = w8 + wl.C16;
        a.amax = reinterpret_cast<unsigned *>(w8 + wl.amax);
        DART_LAUNCH(launch_sma_bwd_tc(s, a, cs));
        return DART_OK;
    }
    DART_LAUNCH(launch_sma_bwd_delta(s, a, cs));
    DART_LAUNCH(launch_sma_bwd_simt(s, dtype == DART_BF16, a, cs));
    return DART_OK;
}

dart_status dart_sma_bwd_norm(const dart_dims *dims, dart_dtype dtype, float eps, const void *Q, const void *C,
                              const void *E, const void *dH, const float *R, const float *lse, const float *dR,
                              float *dQ, float *dC, float *dE, float *ddH, void *ws, size_t ws_bytes, void *stream) {
    Shape s;
    dart_status st = check_dims(dims, &s);
    if (st != DART_OK) return st;
    if ((st = check_supported(s, dtype)) != DART_OK) return st;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return DART_ERR_DIMS;
    DART_TRY_PTR(Q);
    DART_TRY_PTR(C);
    DART_TRY_PTR(E);
    DART_TRY_PTR(dH);
    DART_OPT_PTR(R);  // not read
    DART_OPT_PTR(lse);
    DART_TRY_PTR(dR);
    DART_TRY_PTR(dQ);
    DART_TRY_PTR(dC);
    DART_TRY_PTR(dE);
    DART_TRY_PTR(ddH);
    if ((st = check_ws(ws, ws_bytes, bwd_norm_ws(s, dtype))) != DART_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    BwdArgs a{};
    a.Q = Q;
    a.C = C;
    a.E = E;
    a.dH = dH;
    a.R = R;
    a.dR = dR;
    if (bwd_tc_shape_ok(s, dtype == DART_BF16)) {
        a.dQ = dQ;
        a.dC = dC;
        a.dE = dE;
        a.ddH = ddH;
        DART_LAUNCH(launch_sma_bwd_norm_tc(s, a, eps, ws, cs));
        return DART_OK;
    }
    // the softmax statistics are recomputed (lse and D into the workspace), so that the gradients do not
    // depend on the precision of the forward that made R and lse
    a.D = static_cast<float *>(ws);
    a.lse_rc = reinterpret_cast<float *>(static_cast<char *>(ws) + bwd_norm_ws(s, dtype) / 2);
    a.lse = a.lse_rc;
    a.dQ = dQ;
    a.dC = dC;
    a.dE = dE;
    a.ddH = ddH;
    DART_LAUNCH(launch_sma_bwd_norm_simt(s, dtype == DART_BF16, a, eps, cs));
    return DART_OK;
}

dart_status dart_layer_fwd(const dart_dims *dims, dart_dtype dtype, const void *X, const void *B, const void *C,
                           const void *Q, const void *E, const float *logA, const float *g, int64_t g_sb,
                           int64_t g_st, int64_t g_sh, void *out, void *dH_out, float *lse_out, void *ws,
                           size_t ws_bytes, void *stream) {
    return dart_layer_fwd_ge(dims, dtype, dims ? dims->nheads : 0, X, B, C, Q, E, logA, g, g_sb, g_st, g_sh, out,
                             dH_out, lse_out, ws, ws_bytes, stream);
}

dart_status dart_layer_fwd_ge(const dart_dims *dims, dart_dtype dtype, int64_t e_groups, const void *X, const void *B,
                              const void *C, const void *Q, const void *E, const float *logA, const float *g,
                              int64_t g_sb, int64_t g_st, int64_t g_sh, void *out, void *dH_out, float *lse_out,
                              void *ws, size_t ws_bytes, void *stream) {
    Shape s;
    dart_status st = check_dims(dims, &s);
    if (st != DART_OK) return st;
    if ((st = check_supported(s, dtype)) != DART_OK) return st;
    if (!e_groups_ok(s, e_groups)) return DART_ERR_DIMS;
    DART_TRY_PTR(X);
    DART_TRY_PTR(B);
    DART_TRY_PTR(C);
    DART_TRY_PTR(Q);
    DART_TRY_PTR(E);
    DART_TRY_PTR(logA);
    if (!g) return DART_ERR_NULL;
    if (!aligned(g, 4)) return DART_ERR_ALIGN;
    if (g_sb < 0 || g_st < 0 || g_sh < 0) return DART_ERR_DIMS;
    DART_TRY_PTR(out);
    DART_TRY_PTR(dH_out);
    DART_OPT_PTR(lse_out);
    if ((st = check_ws(ws, ws_bytes, layer_ws_bytes(s, dtype))) != DART_OK) return st;
    WsLayout w = layer_ws(s, dtype, true);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == DART_BF16;
    LayerPtrs p{};
    p.X = X;
    p.B = B;
    p.C = C;
    p.Q = Q;
    p.E = E;
    p.logA = logA;
    p.g = g;
    p.g_sb = g_sb;
    p.g_st = g_st;
    p.g_sh = g_sh;
    p.dH = dH_out;
    p.Y = out;
    p.R = out;
    p.lse = lse_out;
    p.combine = false;
    p.cs = reinterpret_cast<float *>(static_cast<char *>(ws) + w.cs);
    p.lam = reinterpret_cast<float *>(static_cast<char *>(ws) + w.lam);
    p.Hprev = static_cast<char *>(ws) + w.hprev;
    p.e_groups = e_groups;
    // chunk memories, then the SSD output Y written into out, then the SMA, which adds g R into out (eq 11):
    // R never makes a round trip through HBM
    DART_LAUNCH(launch_chunk_cumsum(s, logA, p.cs, p.lam, cs));
    DART_LAUNCH(launch_chunk_states(s, bf16, p, cs));
    if (use_scan256(s, bf16)) {
        // the scan on 256-token chunks of its own; the SMA reads the S-token chunk memories
        DART_LAUNCH(launch_scan256(s, bf16, p, static_cast<char *>(ws),
                                   scan256_ws(s, dtype, layer_ws(s, dtype, false).total), cs));
    } else {
        DART_LAUNCH(launch_state_pass(s, bf16, p, cs));
        DART_LAUNCH(launch_ssd_out(s, bf16, p, cs));
    }
    p.combine = true;  // gated residual in the SMA epilogue: out = Y + g R
    if (tc_shape_ok_ge(s, bf16, e_groups)) {
        DART_LAUNCH(launch_sma_fwd_tc(s, p, cs));
    } else {
        DART_LAUNCH(launch_sma_fwd_simt(s, bf16, p, cs));
    }
    return DART_OK;
}

static dart_status decode_check(int64_t batch, int64_t nheads, int64_t ngroups, int64_t dstate, int64_t headdim,
                                int64_t n_chunks, int64_t chunk_stride, dart_dtype dtype) {
    if (dtype != DART_F32 && dtype != DART_BF16) return DART_ERR_DTYPE;
    if (batch <= 0 || nheads <= 0 || ngroups <= 0 || dstate <= 0 || headdim <= 0 || n_chunks < 0 ||
        chunk_stride < n_chunks || chunk_stride <= 0)
        return DART_ERR_DIMS;
    if (nheads % ngroups != 0 || batch > kMaxGrid || nheads > kMaxGrid) return DART_ERR_DIMS;
    if (dstate > 256) return DART_ERR_UNSUPPORTED;
    const int64_t row_bytes = headdim * (int64_t)esize(dtype);
    if (row_bytes % 16 != 0) return DART_ERR_UNSUPPORTED;
    const int64_t vpr = row_bytes / 16;
    if (vpr > 32 || (vpr & (vpr - 1)) != 0) return DART_ERR_UNSUPPORTED;
    return DART_OK;
}

size_t dart_decode_workspace_size(int64_t batch, int64_t nheads, int64_t dstate, int64_t headdim, int64_t n_chunks,
                                  dart_dtype dtype) {
    if (decode_check(batch, nheads, 1, dstate, headdim, n_chunks, n_chunks > 0 ? n_chunks : 1, dtype) != DART_OK)
        return 0;
    int splits = decode_splits(batch, nheads, n_chunks);
    return round_up((size_t)(batch * nheads * splits * (2 + headdim)) * sizeof(float), 256);
}

dart_status dart_sma_decode(int64_t batch, int64_t nheads, int64_t ngroups, int64_t dstate, int64_t headdim,
                            int64_t n_chunks, int64_t chunk_stride, dart_dtype dtype, const void *Q, const void *C,
                            const void *E, const void *Y, const float *g, int64_t g_sb, int64_t g_sh,
                            const void *cache, void *out, float *lse, void *ws, size_t ws_bytes, void *stream) {
    return dart_sma_decode_ge(batch, nheads, ngroups, nheads, dstate, headdim, n_chunks, chunk_stride, dtype, Q, C, E,
                              Y, g, g_sb, g_sh, cache, out, lse, ws, ws_bytes, stream);
}

dart_status dart_sma_decode_ge(int64_t batch, int64_t nheads, int64_t ngroups, int64_t e_groups, int64_t dstate,
                               int64_t headdim, int64_t n_chunks, int64_t chunk_stride, dart_dtype dtype,
                               const void *Q, const void *C, const void *E, const void *Y, const float *g,
                               int64_t g_sb, int64_t g_sh, const void *cache, void *out, float *lse, void *ws,
                               size_t ws_bytes, void *stream) {
    dart_status st = decode_check(batch, nheads, ngroups, dstate, headdim, n_chunks, chunk_stride, dtype);
    if (st != DART_OK) return st;
    if (e_groups < 1 || e_groups > nheads || nheads % e_groups != 0) return DART_ERR_DIMS;
    DART_TRY_PTR(Q);
    DART_TRY_PTR(C);
    DART_TRY_PTR(E);
    DART_TRY_PTR(Y);
    if (!g) return DART_ERR_NULL;
    if (!aligned(g, 4)) return DART_ERR_ALIGN;
    if (g_sb < 0 || g_sh < 0) return DART_ERR_DIMS;
    DART_TRY_PTR(cache);
    DART_TRY_PTR(out);
    DART_OPT_PTR(lse);
    size_t need = dart_decode_workspace_size(batch, nheads, dstate, headdim, n_chunks, dtype);
    if ((st = check_ws(ws, ws_bytes, need)) != DART_OK) return st;
    DecodeArgs a{};
    a.Bt = batch;
    a.H = nheads;
    a.G = ngroups;
    a.N = dstate;
    a.P = headdim;
    a.n_chunks = n_chunks;
    a.chunk_stride = chunk_stride;
    a.Q = Q;
    a.C = C;
    a.E = E;
    a.Y = Y;
    a.g = g;
    a.g_sb = g_sb;
    a.g_sh = g_sh;
    a.cache = cache;
    a.out = out;
    a.lse = lse;
    a.partials = static_cast<float *>(ws);
    a.splits = decode_splits(batch, nheads, n_chunks);
    a.EG = e_groups;
    DART_LAUNCH(launch_sma_decode(a, dtype == DART_BF16, static_cast<cudaStream_t>(stream)));
    return DART_OK;
}

size_t dart_decode_step_workspace_size(int64_t batch, int64_t nheads, int64_t dstate, int64_t headdim,
                                       int64_t n_chunks, dart_dtype dtype) {
    const size_t part = dart_decode_workspace_size(batch, nheads, dstate, headdim, n_chunks, dtype);
    if (part == 0) return 0;
    return round_up((size_t)(batch * nheads * headdim) * sizeof(float), 256) + part;
}

dart_status dart_decode_step(int64_t batch, int64_t nheads, int64_t ngroups, int64_t dstate, int64_t headdim,
                             int64_t n_chunks, int64_t chunk_stride, int close_chunk, dart_dtype dtype,
                             const void *X, const void *B, const void *C, const void *Q, const void *E,
                             const float *logA, const float *g, int64_t g_sb, int64_t g_sh, float *state,
                             float *chunk_acc, void *cache, void *out, float *lse, void *ws, size_t ws_bytes,
                             void *stream) {
    dart_status st = decode_check(batch, nheads, ngroups, dstate, headdim, n_chunks, chunk_stride, dtype);
    if (st != DART_OK) return st;
    if (close_chunk && n_chunks >= chunk_stride) return DART_ERR_DIMS;  // no free slot for the closing chunk
    DART_TRY_PTR(X);
    DART_TRY_PTR(B);
    DART_TRY_PTR(C);
    DART_TRY_PTR(Q);
    DART_TRY_PTR(E);
    if (!logA || !g) return DART_ERR_NULL;
    if (!aligned(logA, 4) || !aligned(g, 4)) return DART_ERR_ALIGN;
    if (g_sb < 0 || g_sh < 0) return DART_ERR_DIMS;
    DART_TRY_PTR(state);
    DART_TRY_PTR(chunk_acc);
    DART_TRY_PTR(cache);
    DART_TRY_PTR(out);
    DART_OPT_PTR(lse);
    size_t need = dart_decode_step_workspace_size(batch, nheads, dstate, headdim, n_chunks, dtype);
    if ((st = check_ws(ws, ws_bytes, need)) != DART_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    float *Yw = static_cast<float *>(ws);
    const size_t y_bytes = round_up((size_t)(batch * nheads * headdim) * sizeof(float), 256);
    StateStepArgs sa{};
    sa.Bt = batch;
    sa.H = nheads;
    sa.G = ngroups;
    sa.N = dstate;
    sa.P = headdim;
    sa.n_chunks = n_chunks;
    sa.chunk_stride = chunk_stride;
    sa.close_chunk = close_chunk ? 1 : 0;
    sa.X = X;
    sa.B = B;
    sa.C = C;
    sa.logA = logA;
    sa.state = state;
    sa.acc = chunk_acc;
    sa.cache = cache;
    sa.Y = Yw;
    DART_LAUNCH(launch_decode_state(sa, dtype == DART_BF16, cs));
    // the readout reads cache slots [0, n_chunks) only; the slot the step may have filled is n_chunks
    DecodeArgs a{};
    a.Bt = batch;
    a.H = nheads;
    a.G = ngroups;
    a.N = dstate;
    a.P = headdim;
    a.n_chunks = n_chunks;
    a.chunk_stride = chunk_stride;
    a.Q = Q;
    a.C = C;
    a.E = E;
    a.Y = Yw;
    a.y_f32 = true;
    a.g = g;
    a.g_sb = g_sb;
    a.g_sh = g_sh;
    a.cache = cache;
    a.out = out;
    a.lse = lse;
    a.partials = reinterpret_cast<float *>(static_cast<char *>(ws) + y_bytes);
    a.splits = decode_splits(batch, nheads, n_chunks);
    DART_LAUNCH(launch_sma_decode(a, dtype == DART_BF16, cs));
    return DART_OK;
}

int dart_device_error(void) { return read_device_error(true); }

dart_status dart_set_wait_limit(uint64_t ns) {
    if (ns > 10000000000ull) return DART_ERR_DIMS;
    const cudaError_t e = set_wait_limit_ns(ns == 0 ? 2000000000ull : ns);
    if (e != cudaSuccess) {
        set_last_error("cudaMemcpyToSymbol(wait limit)", e);
        return DART_ERR_CUDA;
    }
    return DART_OK;
}

int dart_fp16_range_flags(void) { return read_fp16_range(true); }

const char *dart_last_error(void) { return last_error(); }

int64_t dart_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int dart_kernel_kinds(void) { return KK_COUNT; }

const char *dart_kernel_name(int id) { return kernel_name(id); }

dart_status dart_profile_enable(int enable) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_profile = enable != 0;
    return DART_OK;
}

dart_status dart_profile_read(int id, double *total_ms, int64_t *launches) {
    if (id < 0 || id >= KK_COUNT) return DART_ERR_DIMS;
    if (!total_ms || !launches) return DART_ERR_NULL;
    std::lock_guard<std::mutex> lk(g_mu);
    double sum = 0.0;
    for (const Rec &r : g_recs[id]) {
        if (cudaEventSynchronize(r.b) != cudaSuccess) return DART_ERR_CUDA;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return DART_ERR_CUDA;
        sum += ms;
    }
    *total_ms = sum;
    *launches = (int64_t)g_recs[id].size();
    return DART_OK;
}

dart_status dart_profile_reset(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (int k = 0; k < KK_COUNT; ++k) {
        for (const Rec &r : g_recs[k]) {
            cudaEventSynchronize(r.b);
            cudaEventDestroy(r.a);
            cudaEventDestroy(r.b);
        }
        g_recs[k].clear();
    }
    return DART_OK;
}

}  // extern "C"
