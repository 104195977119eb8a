// CUDA-core kernels of the DART forward path.
//
// These run every supported shape (N <= 256, P <= 256, N*P <= 16384, S <= 1024)
// in fp32 arithmetic for fp32 or bf16 storage. The bf16 / N=128 / P=64 shapes of
// the paper's kernel setting (§5.3) take the tcgen05 kernels instead where one
// exists; the chunk cumsum, the state-passing recurrence and the decode kernel
// below serve both paths.
#include <math.h>
#include <string.h>

#include "dart_internal.cuh"

namespace dart {

namespace {

constexpr int kThreads = 256;
constexpr float kNegInf = -INFINITY;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

template <typename T>
__device__ __forceinline__ float ldf(const T *p) {
    return to_f32(p[0]);
}

// ---------------------------------------------------------------------------
// a1: within-chunk inclusive cumsum of logA and chunk totals.
//   cs[b, h, t] = sum_{r = chunk start}^{t} logA[b, r, h]   (eq 3 / eq 16 as log-sums)
//   lam[b, h, c] = cs at the last token of chunk c
// grid (M, ceil(H / HB), Bt); a warp scans one head of the chunk at a time.
// ---------------------------------------------------------------------------
// Tile layout: head hh's tokens at tile[hh * pitch + tt + tt / 8], pitch = S + S / 8 + 1 (odd). The
// load (consecutive threads = consecutive heads) and the scan (lane = 8 consecutive tokens) both hit
// 32 distinct banks.
__host__ __device__ __forceinline__ int cumsum_pitch(int64_t S) { return (int)(S + S / 8 + 1); }

__global__ void __launch_bounds__(kThreads) k_chunk_cumsum(Shape s, int HB, const float *__restrict__ logA,
                                                           float *__restrict__ cs, float *__restrict__ lam) {
    extern __shared__ float tile[];  // [HB][pitch]
    const int c = blockIdx.x;
    const int64_t h0 = (int64_t)blockIdx.y * HB;
    const int64_t b = blockIdx.z;
    const int hb = (int)min((int64_t)HB, s.H - h0);
    const int64_t t0 = (int64_t)c * s.S;
    const int len = (int)min(s.S, s.L - t0);
    const int pitch = cumsum_pitch(s.S);
    // every load of the tile is issued before the first shared-memory store that consumes one
    constexpr int kPer = 8;  // elements per thread when S * HB <= kPer * blockDim.x
    const int n = len * hb;
    float v[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int i = threadIdx.x + q * (int)blockDim.x;
        const int tt = i / hb, hh = i - tt * hb;
        v[q] = i < n ? logA[(b * s.L + t0 + tt) * s.H + h0 + hh] : 0.f;
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int i = threadIdx.x + q * (int)blockDim.x;
        const int tt = i / hb, hh = i - tt * hb;
        if (i < n) tile[hh * pitch + tt + (tt >> 3)] = v[q];
    }
    for (int i = threadIdx.x + kPer * (int)blockDim.x; i < n; i += blockDim.x) {  // larger tiles only
        const int tt = i / hb, hh = i - tt * hb;
        tile[hh * pitch + tt + (tt >> 3)] = logA[(b * s.L + t0 + tt) * s.H + h0 + hh];
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per = (len + 31) / 32;
    for (int hh = warp; hh < hb; hh += blockDim.x / 32) {
        const float *th = tile + hh * pitch;
        int beg = min(len, lane * per), end = min(len, beg + per);
        float run = 0.f;
        for (int tt = beg; tt < end; ++tt) run += th[tt + (tt >> 3)];
        float incl = run;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            float v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        float acc = incl - run;
        float *dst = cs + (b * s.H + h0 + hh) * s.L + t0;
        for (int tt = beg; tt < end; ++tt) {
            acc += th[tt + (tt >> 3)];
            dst[tt] = acc;
        }
        if (lane == 31) lam[(b * s.H + h0 + hh) * s.M + c] = incl;
    }
}

// ---------------------------------------------------------------------------
// a2: chunk state memories, eq (5): dH[c][n, p] = sum_s w_s B_s[n] X_s[p],
//     w_s = exp(lam_c - cs_s) = A_{s+1:e(c)}.
// grid (M * nsplit, H, Bt); each thread owns up to 32 (n, p) outputs.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads) k_chunk_states_simt(Shape s, int nsplit, const T *__restrict__ X,
                                                                const T *__restrict__ B, const float *__restrict__ cs,
                                                                const float *__restrict__ lam, T *__restrict__ dH) {
    constexpr int OPT = 32, SB = 32;
    extern __shared__ float sm[];
    const int c = blockIdx.x / nsplit, split = blockIdx.x % nsplit;
    const int64_t h = blockIdx.y, b = blockIdx.z;
    const int64_t g = h / (s.H / s.G);
    const int64_t t0 = (int64_t)c * s.S;
    const int len = (int)min(s.S, s.L - t0);
    const int N = (int)s.N, P = (int)s.P;
    float *w = sm;
    float *Bs = w + s.S;       // [SB][N]
    float *Xs = Bs + SB * N;   // [SB][P]
    const float *csb = cs + (b * s.H + h) * s.L + t0;
    const float total = lam[(b * s.H + h) * s.M + c];
    for (int i = threadIdx.x; i < len; i += blockDim.x) w[i] = expf(total - csb[i]);
    const int NP = N * P;
    const int base = split * kThreads * OPT;
    float acc[OPT];
#pragma unroll
    for (int k = 0; k < OPT; ++k) acc[k] = 0.f;
    for (int s0 = 0; s0 < len; s0 += SB) {
        const int nb = min(SB, len - s0);
        __syncthreads();
        for (int i = threadIdx.x; i < nb * N; i += blockDim.x) {
            int r = i / N, n = i % N;
            Bs[r * N + n] = ldf(B + ((b * s.L + t0 + s0 + r) * s.G + g) * N + n);
        }
        for (int i = threadIdx.x; i < nb * P; i += blockDim.x) {
            int r = i / P, p = i % P;
            Xs[r * P + p] = ldf(X + ((b * s.L + t0 + s0 + r) * s.H + h) * P + p) * w[s0 + r];
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < OPT; ++k) {
            int idx = base + threadIdx.x + kThreads * k;
            if (idx < NP) {
                int n = idx / P, p = idx % P;
                float a = acc[k];
                for (int r = 0; r < nb; ++r) a = fmaf(Bs[r * N + n], Xs[r * P + p], a);
                acc[k] = a;
            }
        }
    }
    T *dst = dH + ((b * s.H + h) * s.M + c) * (int64_t)NP;
#pragma unroll
    for (int k = 0; k < OPT; ++k) {
        int idx = base + threadIdx.x + kThreads * k;
        if (idx < NP) dst[idx] = from_f32<T>(acc[k]);
    }
}

// ---------------------------------------------------------------------------
// a3: chunk-boundary state passing, App. A eq (18):
//     H_[c] = exp(lam_c) H_[c-1] + dH[c],  H_[-1] = 0;  Hprev[c] = H_[c-1].
// Each thread owns one 16-byte vector of one (b, h) state (8 bf16 or 4 fp32
// elements) and runs the recurrence over the chunks in order, with the loads of
// the next kDepth chunks in flight. A warp's loads and stores are 512 contiguous
// bytes of one chunk memory. grid (ceil(NP / (256 V)), H, Bt).
// ---------------------------------------------------------------------------
// 16 bytes of chunk c (zeros past the last chunk); the ragged edge of a state (nv < V elements) is
// read element by element, with compile-time indices so that nothing leaves registers.
template <typename T>
__device__ __forceinline__ uint4 state_pass_load(const T *src, int64_t c, int64_t M, int64_t NP, int nv, bool vec) {
    constexpr int V = 16 / sizeof(T);
    if (c >= M) return make_uint4(0u, 0u, 0u, 0u);
    if (vec) return __ldg(reinterpret_cast<const uint4 *>(src + c * NP));
    T el[V];
#pragma unroll
    for (int j = 0; j < V; ++j) el[j] = j < nv ? src[c * NP + j] : from_f32<T>(0.f);
    uint4 v;
    memcpy(&v, el, sizeof(v));
    return v;
}

// Four resident blocks per SM (at most 64 registers a thread) keep the whole grid of a layer-sized
// problem in one wave; each thread keeps kDepth chunk loads in flight, reissuing a slot's load as
// soon as the slot is consumed.
template <typename T>
__global__ void __launch_bounds__(kThreads, 4) k_state_pass(Shape s, const T *__restrict__ dH,
                                                            const float *__restrict__ lam, T *__restrict__ Hprev,
                                                            float *__restrict__ final_state) {
    constexpr int V = 16 / sizeof(T);
    constexpr int kDepth = 6;
    extern __shared__ float decay[];  // [M] exp(lam_c)
    const int64_t bh = (int64_t)blockIdx.z * s.H + blockIdx.y;
    for (int64_t c = threadIdx.x; c < s.M; c += blockDim.x) decay[c] = expf(lam[bh * s.M + c]);
    __syncthreads();
    const int64_t NP = s.N * s.P;
    const int64_t e0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * V;
    if (e0 >= NP) return;
    const T *src = dH + bh * s.M * NP + e0;
    T *dst = Hprev + bh * s.M * NP + e0;
    const int nv = (int)min((int64_t)V, NP - e0);
    const bool vec = (nv == V) && ((NP * (int64_t)sizeof(T)) % 16 == 0);
    float h[V];
#pragma unroll
    for (int j = 0; j < V; ++j) h[j] = 0.f;
    uint4 buf[kDepth];
#pragma unroll
    for (int d = 0; d < kDepth; ++d) buf[d] = state_pass_load(src, d, s.M, NP, nv, vec);
    for (int64_t c0 = 0; c0 < s.M; c0 += kDepth) {
#pragma unroll
        for (int d = 0; d < kDepth; ++d) {
            const int64_t c = c0 + d;
            if (c >= s.M) break;
            T x[V];
            memcpy(x, &buf[d], sizeof(x));
            buf[d] = state_pass_load(src, c + kDepth, s.M, NP, nv, vec);
            T o[V];
            const float a = decay[c];
#pragma unroll
            for (int j = 0; j < V; ++j) {
                o[j] = from_f32<T>(h[j]);  // state entering chunk c
                h[j] = fmaf(a, h[j], to_f32(x[j]));
            }
            if (vec) {
                uint4 outv;
                memcpy(&outv, o, sizeof(outv));
                *reinterpret_cast<uint4 *>(dst + c * NP) = outv;
            } else {
#pragma unroll
                for (int j = 0; j < V; ++j)
                    if (j < nv) dst[c * NP + j] = o[j];
            }
        }
    }
    if (final_state) {
#pragma unroll
        for (int j = 0; j < V; ++j)
            if (j < nv) final_state[bh * NP + e0 + j] = h[j];
    }
}

// ---------------------------------------------------------------------------
// a4: SSD output, App. A eq (21)-(22):
//   Y_t = sum_{s in c, s <= t} (C_t . B_s) exp(cs_t - cs_s) X_s + exp(cs_t) C_t Hprev[c]
// grid (M * ntile, H, Bt), TT = 32 tokens per block.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads) k_ssd_out_simt(Shape s, int ntile, const T *__restrict__ X,
                                                           const T *__restrict__ B, const T *__restrict__ C,
                                                           const float *__restrict__ cs, const T *__restrict__ Hprev,
                                                           float *__restrict__ Y) {
    constexpr int TT = 32, SB = 32, OPT = 32;
    extern __shared__ float sm[];
    const int N = (int)s.N, P = (int)s.P, NB = N + 1;
    const int c = blockIdx.x / ntile, tile = blockIdx.x % ntile;
    const int64_t h = blockIdx.y, b = blockIdx.z;
    const int64_t g = h / (s.H / s.G);
    const int64_t tc0 = (int64_t)c * s.S;
    const int64_t t0 = tc0 + (int64_t)tile * TT;
    const int64_t tlim = min(s.L, tc0 + s.S);
    if (t0 >= tlim) return;
    const int tlen = (int)min((int64_t)TT, tlim - t0);
    float *Cs = sm;                 // [TT][N]
    float *Bs = Cs + TT * N;        // [SB][N + 1]
    float *Xs = Bs + SB * NB;       // [SB][P]   (also Hprev rows)
    float *Gs = Xs + SB * P;        // [TT][SB]
    float *cst = Gs + TT * SB;      // [TT]
    float *css = cst + TT;          // [SB]
    const float *csb = cs + (b * s.H + h) * s.L;
    for (int i = threadIdx.x; i < TT * N; i += blockDim.x) {
        int r = i / N, n = i % N;
        Cs[i] = r < tlen ? ldf(C + ((b * s.L + t0 + r) * s.G + g) * N + n) : 0.f;
    }
    for (int i = threadIdx.x; i < TT; i += blockDim.x) cst[i] = i < tlen ? csb[t0 + i] : 0.f;
    float acc[OPT];
#pragma unroll
    for (int k = 0; k < OPT; ++k) acc[k] = 0.f;
    for (int64_t sb0 = tc0; sb0 < t0 + tlen; sb0 += SB) {
        const int nb = (int)min((int64_t)SB, t0 + tlen - sb0);
        __syncthreads();
        for (int i = threadIdx.x; i < nb * N; i += blockDim.x) {
            int r = i / N, n = i % N;
            Bs[r * NB + n] = ldf(B + ((b * s.L + sb0 + r) * s.G + g) * N + n);
        }
        for (int i = threadIdx.x; i < nb * P; i += blockDim.x) {
            int r = i / P, p = i % P;
            Xs[r * P + p] = ldf(X + ((b * s.L + sb0 + r) * s.H + h) * P + p);
        }
        for (int i = threadIdx.x; i < nb; i += blockDim.x) css[i] = csb[sb0 + i];
        __syncthreads();
        for (int q = threadIdx.x; q < TT * SB; q += blockDim.x) {
            int i = q / SB, j = q % SB;
            float v = 0.f;
            if (i < tlen && j < nb && sb0 + j <= t0 + i) {
                float d = 0.f;
                for (int n = 0; n < N; ++n) d = fmaf(Cs[i * N + n], Bs[j * NB + n], d);
                v = d * expf(cst[i] - css[j]);
            }
            Gs[q] = v;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < OPT; ++k) {
            int idx = threadIdx.x + kThreads * k;
            int i = idx / P, p = idx % P;
            if (i < tlen) {
                float a = acc[k];
                for (int j = 0; j < nb; ++j) a = fmaf(Gs[i * SB + j], Xs[j * P + p], a);
                acc[k] = a;
            }
        }
    }
    if (c > 0) {
        float acc2[OPT];
#pragma unroll
        for (int k = 0; k < OPT; ++k) acc2[k] = 0.f;
        const T *Hp = Hprev + ((b * s.H + h) * s.M + c) * (int64_t)N * P;
        for (int n0 = 0; n0 < N; n0 += SB) {
            const int nb = min(SB, N - n0);
            __syncthreads();
            for (int i = threadIdx.x; i < nb * P; i += blockDim.x) Xs[i] = ldf(Hp + (int64_t)n0 * P + i);
            __syncthreads();
#pragma unroll
            for (int k = 0; k < OPT; ++k) {
                int idx = threadIdx.x + kThreads * k;
                int i = idx / P, p = idx % P;
                if (i < tlen) {
                    float a = acc2[k];
                    for (int j = 0; j < nb; ++j) a = fmaf(Cs[i * N + n0 + j], Xs[j * P + p], a);
                    acc2[k] = a;
                }
            }
        }
#pragma unroll
        for (int k = 0; k < OPT; ++k) {
            int idx = threadIdx.x + kThreads * k;
            int i = idx / P;
            if (i < tlen) acc[k] = fmaf(expf(cst[i]), acc2[k], acc[k]);
        }
    }
#pragma unroll
    for (int k = 0; k < OPT; ++k) {
        int idx = threadIdx.x + kThreads * k;
        int i = idx / P, p = idx % P;
        if (i < tlen) {
            Y[((b * s.L + t0 + i) * s.H + h) * P + p] = acc[k];
        }
    }
}

// ---------------------------------------------------------------------------
// a5/a6: state-memory attention, eq (8)-(10), online softmax (App. C eq 28-31),
// optional gated residual (eq 11) in the epilogue. With prm.score_norm, the
// normalised score branch of App. B.1 eq (25)-(27): Q_t and E_t divided by their
// RMS, and each chunk memory's row n weighted by r_n = (mean_p dH_np^2 + eps)^-1/2
// on the key side only.
// grid (M * ntile, H, Bt), TT = 16 tokens per block, 2 tokens per warp; lane
// owns p = lane + 32 k.
// ---------------------------------------------------------------------------
template <typename T, int KP>
__global__ void __launch_bounds__(kThreads) k_sma_fwd_simt(Shape s, int ntile, LayerPtrs prm) {
    constexpr int TT = 16;
    extern __shared__ float sm[];
    const T *__restrict__ Q = static_cast<const T *>(prm.Q);
    const T *__restrict__ Cp = static_cast<const T *>(prm.C);
    const T *__restrict__ E = static_cast<const T *>(prm.E);
    const T *__restrict__ dH = static_cast<const T *>(prm.dH);
    const int N = (int)s.N, P = (int)s.P;
    const int64_t hpe = heads_per_e(s, prm.e_groups), eg = s.H / hpe;  // E groups and heads per group
    const int c = blockIdx.x / ntile, tile = blockIdx.x % ntile;
    const int64_t h = blockIdx.y, b = blockIdx.z;
    const int64_t g = h / (s.H / s.G);
    const int64_t tc0 = (int64_t)c * s.S;
    const int64_t t0 = tc0 + (int64_t)tile * TT;
    const int64_t tlim = min(s.L, tc0 + s.S);
    if (t0 >= tlim) return;
    const int tlen = (int)min((int64_t)TT, tlim - t0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (c == 0) {  // no historical chunk: R = 0, lse = -inf; the combine adds nothing
        for (int tk = 0; tk < 2; ++tk) {
            int tl = warp * 2 + tk;
            if (tl >= tlen) continue;
            int64_t t = t0 + tl;
            if (!prm.combine) {
                float *Rr = static_cast<float *>(prm.R) + ((b * s.L + t) * s.H + h) * P;
                for (int p = lane; p < P; p += 32) Rr[p] = 0.f;
            }
            if (prm.lse && lane == 0) prm.lse[(b * s.H + h) * s.L + t] = kNegInf;
        }
        return;
    }
    float *Qs = sm;            // [TT][N]
    float *Cs = Qs + TT * N;   // [TT][N]
    float *Hs = Cs + TT * N;   // [N][P]
    float *Rn = Hs + N * P;    // [N] row weights of the normalised branch
    const bool norm = prm.score_norm;
    const float eps = prm.norm_eps;
    for (int i = threadIdx.x; i < TT * N; i += blockDim.x) {
        int r = i / N, n = i % N;
        bool ok = r < tlen;
        Qs[i] = ok ? ldf(Q + ((b * s.L + t0 + r) * s.G + g) * N + n) : 0.f;
        Cs[i] = ok ? ldf(Cp + ((b * s.L + t0 + r) * s.G + g) * N + n) : 0.f;
    }
    if (norm) {  // Q_t / RMS(Q_t), eq (25): each warp its two rows
        __syncthreads();
#pragma unroll
        for (int tk = 0; tk < 2; ++tk) {
            const int tl = warp * 2 + tk;
            float sq = 0.f;
            for (int n = lane; n < N; n += 32) sq = fmaf(Qs[tl * N + n], Qs[tl * N + n], sq);
            const float inv = rsqrtf(warp_sum(sq) / (float)N + eps);
            for (int n = lane; n < N; n += 32) Qs[tl * N + n] *= inv;
        }
    }
    const float scale = rsqrtf((float)N);
    float Ev[2][KP], O[2][KP], m[2], d[2];
#pragma unroll
    for (int tk = 0; tk < 2; ++tk) {
        int tl = warp * 2 + tk;
        m[tk] = kNegInf;
        d[tk] = 0.f;
#pragma unroll
        for (int k = 0; k < KP; ++k) {
            int p = lane + 32 * k;
            Ev[tk][k] = (tl < tlen && p < P) ? ldf(E + ((b * s.L + t0 + tl) * eg + h / hpe) * P + p) * scale : 0.f;
            O[tk][k] = 0.f;
        }
        if (norm) {  // E_t / RMS(E_t), eq (25) (the 1/sqrt(N) above is a common factor)
            float sq = 0.f;
#pragma unroll
            for (int k = 0; k < KP; ++k) sq = fmaf(Ev[tk][k], Ev[tk][k], sq);
            const float inv = rsqrtf(warp_sum(sq) / (scale * scale * (float)P) + eps);
#pragma unroll
            for (int k = 0; k < KP; ++k) Ev[tk][k] *= inv;
        }
    }
    const T *dHb = dH + (b * s.H + h) * s.M * (int64_t)N * P;
    for (int j = 0; j < c; ++j) {
        __syncthreads();
        const T *src = dHb + (int64_t)j * N * P;
        for (int i = threadIdx.x; i < N * P; i += blockDim.x) Hs[i] = ldf(src + i);
        __syncthreads();
        if (norm) {  // r_n of this chunk memory, eq (26)
            for (int n = threadIdx.x; n < N; n += blockDim.x) {
                float sq = 0.f;
                for (int p = 0; p < P; ++p) sq = fmaf(Hs[n * P + p], Hs[n * P + p], sq);
                Rn[n] = rsqrtf(sq / (float)P + eps);
            }
            __syncthreads();
        }
#pragma unroll
        for (int tk = 0; tk < 2; ++tk) {
            int tl = warp * 2 + tk;
            if (tl >= tlen) continue;
            float u[KP], v[KP];
#pragma unroll
            for (int k = 0; k < KP; ++k) u[k] = v[k] = 0.f;
            for (int n = 0; n < N; ++n) {
                float qn = norm ? Qs[tl * N + n] * Rn[n] : Qs[tl * N + n], cn = Cs[tl * N + n];
#pragma unroll
                for (int k = 0; k < KP; ++k) {
                    int p = lane + 32 * k;
                    float hv = p < P ? Hs[n * P + p] : 0.f;
                    u[k] = fmaf(qn, hv, u[k]);
                    v[k] = fmaf(cn, hv, v[k]);
                }
            }
            float l = 0.f;
#pragma unroll
            for (int k = 0; k < KP; ++k) l = fmaf(u[k], Ev[tk][k], l);
            l = warp_sum(l);
            float mn = fmaxf(m[tk], l);
            float alpha = expf(m[tk] - mn);
            float pw = expf(l - mn);
            d[tk] = fmaf(d[tk], alpha, pw);
#pragma unroll
            for (int k = 0; k < KP; ++k) O[tk][k] = fmaf(O[tk][k], alpha, pw * v[k]);
            m[tk] = mn;
        }
    }
#pragma unroll
    for (int tk = 0; tk < 2; ++tk) {
        int tl = warp * 2 + tk;
        if (tl >= tlen) continue;
        int64_t t = t0 + tl;
        float inv = 1.f / d[tk];
        int64_t row = ((b * s.L + t) * s.H + h) * P;
        if (prm.combine) {
            float gv = prm.g[b * prm.g_sb + t * prm.g_st + h * prm.g_sh];
            float *Yr = static_cast<float *>(prm.Y) + row;
#pragma unroll
            for (int k = 0; k < KP; ++k) {
                int p = lane + 32 * k;
                if (p < P) Yr[p] = fmaf(gv, O[tk][k] * inv, Yr[p]);
            }
        } else {
            float *Rr = static_cast<float *>(prm.R) + row;
#pragma unroll
            for (int k = 0; k < KP; ++k) {
                int p = lane + 32 * k;
                if (p < P) Rr[p] = O[tk][k] * inv;
            }
        }
        if (prm.lse && lane == 0) prm.lse[(b * s.H + h) * s.L + t] = m[tk] + logf(d[tk]);
    }
}

// ---------------------------------------------------------------------------
// a7: single-token decode over cached chunk memories (bandwidth-bound).
// Each warp streams whole chunks with 128-bit loads: lane owns one 16-byte
// column vector (pv) of every RPP-th row. Per chunk it forms
//   l = sum_n Q_n sum_p dH[n,p] E_p / sqrt(N)   and   V_p = sum_n C_n dH[n,p],
// then folds (l, V) into its online-softmax state. Warps are merged in shared
// memory and the CTA writes one (m, d, O[P]) partial per chunk split.
// grid (splits, H, Bt), 8 warps per block.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void unpack16(const uint4 &raw, float (&x)[8], const __nv_bfloat16 *) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void unpack16(const uint4 &raw, float (&x)[4], const float *) {
    x[0] = __uint_as_float(raw.x);
    x[1] = __uint_as_float(raw.y);
    x[2] = __uint_as_float(raw.z);
    x[3] = __uint_as_float(raw.w);
}

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

template <typename T, int VPR>
__global__ void __launch_bounds__(kThreads) k_sma_decode(DecodeArgs a, int64_t per_split) {
    constexpr int EPV = 16 / sizeof(T);  // elements per 16-byte vector
    constexpr int RPP = 32 / VPR;        // rows per warp pass
    constexpr int UNR = 8;               // 16-byte loads in flight per lane
    constexpr int NW = kThreads / 32;
    extern __shared__ float sm[];
    const int N = (int)a.N, P = (int)a.P;
    float *Qs = sm;                // [N]
    float *Cs = Qs + N;            // [N]
    float *wm = Cs + N;            // [NW]
    float *wd = wm + NW;           // [NW]
    float *wO = wd + NW;           // [NW][P]
    const int split = blockIdx.x;
    const int64_t h = blockIdx.y, b = blockIdx.z;
    const int64_t grp = h / (a.H / a.G);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const T *Qp = static_cast<const T *>(a.Q) + (b * a.G + grp) * N;
    const T *Cp = static_cast<const T *>(a.C) + (b * a.G + grp) * N;
    const float scale = rsqrtf((float)N);
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
        Qs[i] = to_f32(Qp[i]) * scale;
        Cs[i] = to_f32(Cp[i]);
    }
    __syncthreads();
    const int pv = lane % VPR, r0 = lane / VPR;
    float Ev[EPV];
    {
        const int64_t eg = a.EG > 0 ? a.EG : a.H;  // E groups; head h reads group h / (H / EG)
        const T *Ep = static_cast<const T *>(a.E) + (b * eg + h / (a.H / eg)) * P + pv * EPV;
#pragma unroll
        for (int e = 0; e < EPV; ++e) Ev[e] = to_f32(Ep[e]);
    }
    float m = kNegInf, d = 0.f, O[EPV];
#pragma unroll
    for (int e = 0; e < EPV; ++e) O[e] = 0.f;
    const int64_t c_begin = (int64_t)split * per_split;
    const int64_t c_end = min(a.n_chunks, c_begin + per_split);
    const int64_t NP = (int64_t)N * P;
    const T *cache = static_cast<const T *>(a.cache) + ((b * a.H + h) * a.chunk_stride) * NP;
    const int passes = (N + RPP - 1) / RPP;
    for (int64_t c = c_begin + warp; c < c_end; c += NW) {
        const uint4 *base = reinterpret_cast<const uint4 *>(cache + c * NP);
        float l = 0.f, V[EPV];
#pragma unroll
        for (int e = 0; e < EPV; ++e) V[e] = 0.f;
        for (int it0 = 0; it0 < passes; it0 += UNR) {
            uint4 buf[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                int r = (it0 + u) * RPP + r0;
                buf[u] = (it0 + u < passes && r < N) ? ld_stream(base + (int64_t)r * VPR + pv) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                int r = (it0 + u) * RPP + r0;
                if (it0 + u < passes && r < N) {
                    float x[EPV];
                    unpack16(buf[u], x, static_cast<const T *>(nullptr));
                    float dot = 0.f;
#pragma unroll
                    for (int e = 0; e < EPV; ++e) dot = fmaf(x[e], Ev[e], dot);
                    l = fmaf(Qs[r], dot, l);
                    float cn = Cs[r];
#pragma unroll
                    for (int e = 0; e < EPV; ++e) V[e] = fmaf(cn, x[e], V[e]);
                }
            }
        }
        l = warp_sum(l);
#pragma unroll
        for (int off = VPR; off < 32; off <<= 1)
#pragma unroll
            for (int e = 0; e < EPV; ++e) V[e] += __shfl_xor_sync(0xffffffffu, V[e], off);
        float mn = fmaxf(m, l);
        float alpha = expf(m - mn), pw = expf(l - mn);
        d = fmaf(d, alpha, pw);
#pragma unroll
        for (int e = 0; e < EPV; ++e) O[e] = fmaf(O[e], alpha, pw * V[e]);
        m = mn;
    }
    if (r0 == 0) {
#pragma unroll
        for (int e = 0; e < EPV; ++e) wO[warp * P + pv * EPV + e] = O[e];
    }
    if (lane == 0) {
        wm[warp] = m;
        wd[warp] = d;
    }
    __syncthreads();
    float *part = a.partials + ((b * a.H + h) * a.splits + split) * (int64_t)(2 + P);
    float mx = kNegInf;
    for (int w = 0; w < NW; ++w) mx = fmaxf(mx, wm[w]);
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
        float o = 0.f;
        for (int w = 0; w < NW; ++w)
            if (wm[w] != kNegInf) o = fmaf(wO[w * P + p], expf(wm[w] - mx), o);
        part[2 + p] = o;
    }
    if (threadIdx.x == 0) {
        float dd = 0.f;
        for (int w = 0; w < NW; ++w)
            if (wm[w] != kNegInf) dd = fmaf(wd[w], expf(wm[w] - mx), dd);
        part[0] = mx;
        part[1] = dd;
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_decode_merge(DecodeArgs a) {
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / a.H, h = bh % a.H;
    const int P = (int)a.P;
    const float *part = a.partials + bh * a.splits * (int64_t)(2 + P);
    float mx = kNegInf;
    for (int sp = 0; sp < a.splits; ++sp) mx = fmaxf(mx, part[sp * (2 + P)]);
    float dd = 0.f;
    for (int sp = 0; sp < a.splits; ++sp) {
        float ms = part[sp * (2 + P)];
        if (ms != kNegInf) dd = fmaf(part[sp * (2 + P) + 1], expf(ms - mx), dd);
    }
    const float gv = a.g[b * a.g_sb + h * a.g_sh];
    const T *Yp = static_cast<const T *>(a.Y) + bh * P;
    float *outp = static_cast<float *>(a.out) + bh * P;
    const bool empty = !(dd > 0.f);
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
        float o = 0.f;
        if (!empty) {
            for (int sp = 0; sp < a.splits; ++sp) {
                float ms = part[sp * (2 + P)];
                if (ms != kNegInf) o = fmaf(part[sp * (2 + P) + 2 + p], expf(ms - mx), o);
            }
            o /= dd;
        }
        const float yv = a.y_f32 ? static_cast<const float *>(a.Y)[bh * P + p] : to_f32(Yp[p]);
        outp[p] = fmaf(gv, o, yv);
    }
    if (a.lse && threadIdx.x == 0) a.lse[bh] = empty ? kNegInf : mx + logf(dd);
}

// ---------------------------------------------------------------------------
// decode-step state maintenance (eq (2) in recurrent form, one token; §4 "Inference Cache"):
//   state <- a state + B^T X,  acc <- a acc + B^T X (memory of the open chunk),  Y = C state;
//   on a chunk close acc (rounded to T) goes to cache slot n_chunks and acc <- 0.
// grid (H, Bt); thread t owns the 4-column group t % (P/4) of rows t / (P/4) + k * (1024 / P), so a
// warp's loads and stores of state and acc are contiguous float4s; Y's sum over n goes through shared
// memory in a fixed order. P is a power of two in [4, 256] (the decode shapes).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads) k_decode_state(StateStepArgs a) {
    __shared__ float4 red[kThreads];
    const int64_t h = blockIdx.x, b = blockIdx.y, bh = b * a.H + h;
    const int64_t grp = h / (a.H / a.G);
    const int cg = (int)(a.P / 4);          // float4 column groups per row
    const int rows = kThreads / cg;         // rows per pass
    const int c = threadIdx.x % cg, r0 = threadIdx.x / cg;
    const float av = expf(a.logA[bh]);
    const T *Bv = static_cast<const T *>(a.B) + (b * a.G + grp) * a.N;
    const T *Cv = static_cast<const T *>(a.C) + (b * a.G + grp) * a.N;
    const T *Xv = static_cast<const T *>(a.X) + bh * a.P + 4 * c;
    const float x0 = to_f32(Xv[0]), x1 = to_f32(Xv[1]), x2 = to_f32(Xv[2]), x3 = to_f32(Xv[3]);
    float4 *st = reinterpret_cast<float4 *>(a.state + bh * a.N * a.P);
    float4 *ac = reinterpret_cast<float4 *>(a.acc + bh * a.N * a.P);
    T *slot = a.close_chunk ? static_cast<T *>(a.cache) + (bh * a.chunk_stride + a.n_chunks) * a.N * a.P : nullptr;
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t n = r0; n < a.N; n += rows) {
        const int64_t e4 = n * cg + c;
        const float bn = to_f32(Bv[n]), cn = to_f32(Cv[n]);
        const float4 so = st[e4], ao = ac[e4];
        const float4 sn = make_float4(fmaf(av, so.x, bn * x0), fmaf(av, so.y, bn * x1), fmaf(av, so.z, bn * x2),
                                      fmaf(av, so.w, bn * x3));
        const float4 an = make_float4(fmaf(av, ao.x, bn * x0), fmaf(av, ao.y, bn * x1), fmaf(av, ao.z, bn * x2),
                                      fmaf(av, ao.w, bn * x3));
        st[e4] = sn;
        if (slot) {
            T *o = slot + 4 * e4;
            o[0] = from_f32<T>(an.x);
            o[1] = from_f32<T>(an.y);
            o[2] = from_f32<T>(an.z);
            o[3] = from_f32<T>(an.w);
            ac[e4] = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            ac[e4] = an;
        }
        y.x = fmaf(cn, sn.x, y.x);
        y.y = fmaf(cn, sn.y, y.y);
        y.z = fmaf(cn, sn.z, y.z);
        y.w = fmaf(cn, sn.w, y.w);
    }
    red[threadIdx.x] = y;
    __syncthreads();
    if (threadIdx.x < cg) {
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < rows; ++r) {
            const float4 v = red[r * cg + threadIdx.x];
            t.x += v.x;
            t.y += v.y;
            t.z += v.z;
            t.w += v.w;
        }
        reinterpret_cast<float4 *>(a.Y + bh * a.P)[threadIdx.x] = t;
    }
}

inline dim3 grid3(int64_t x, int64_t y, int64_t z) { return dim3((unsigned)x, (unsigned)y, (unsigned)z); }

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

cudaError_t launch_chunk_cumsum(const Shape &s, const float *logA, float *cs, float *lam, cudaStream_t st) {
    // 8 heads of a 256-token chunk per block: 8 tile elements per thread, one head per warp
    int HB = (int)max((int64_t)1, min(s.H, (int64_t)(2048 / s.S)));
    size_t smem = (size_t)cumsum_pitch(s.S) * HB * sizeof(float);
    launch_begin(KK_CHUNK_CUMSUM, st);
    k_chunk_cumsum<<<grid3(s.M, (s.H + HB - 1) / HB, s.Bt), kThreads, smem, st>>>(s, HB, logA, cs, lam);
    return launch_end(KK_CHUNK_CUMSUM, st);
}

template <typename T>
static cudaError_t chunk_states_t(const Shape &s, const LayerPtrs &p, cudaStream_t st) {
    int nsplit = (int)((s.N * s.P + kThreads * 32 - 1) / (kThreads * 32));
    size_t smem = (s.S + 32 * s.N + 32 * s.P) * sizeof(float);
    auto kern = k_chunk_states_simt<T>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_begin(KK_CHUNK_STATES, st);
    kern<<<grid3(s.M * nsplit, s.H, s.Bt), kThreads, smem, st>>>(s, nsplit, static_cast<const T *>(p.X),
                                                                  static_cast<const T *>(p.B), p.cs, p.lam,
                                                                  static_cast<T *>(p.dH));
    return launch_end(KK_CHUNK_STATES, st);
}

cudaError_t launch_chunk_states_simt(const Shape &s, bool bf16, const LayerPtrs &p, cudaStream_t st) {
    return bf16 ? chunk_states_t<__nv_bfloat16>(s, p, st) : chunk_states_t<float>(s, p, st);
}

template <typename T>
static cudaError_t state_pass_t(const Shape &s, const LayerPtrs &p, cudaStream_t st) {
    constexpr int V = 16 / sizeof(T);
    int64_t per_block = (int64_t)kThreads * V;
    int64_t gx = (s.N * s.P + per_block - 1) / per_block;
    size_t smem = (size_t)s.M * sizeof(float);
    auto kern = k_state_pass<T>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_begin(KK_STATE_PASS, st);
    kern<<<grid3(gx, s.H, s.Bt), kThreads, smem, st>>>(s, static_cast<const T *>(p.dH), p.lam,
                                                       static_cast<T *>(p.Hprev), p.final_state);
    return launch_end(KK_STATE_PASS, st);
}

cudaError_t launch_state_pass(const Shape &s, bool bf16, const LayerPtrs &p, cudaStream_t st) {
    return bf16 ? state_pass_t<__nv_bfloat16>(s, p, st) : state_pass_t<float>(s, p, st);
}

template <typename T>
static cudaError_t ssd_out_t(const Shape &s, const LayerPtrs &p, cudaStream_t st) {
    constexpr int TT = 32, SB = 32;
    int ntile = (int)((s.S + TT - 1) / TT);
    size_t smem = (TT * s.N + SB * (s.N + 1) + SB * s.P + TT * SB + TT + SB) * sizeof(float);
    auto kern = k_ssd_out_simt<T>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_begin(KK_SSD_OUT, st);
    kern<<<grid3(s.M * ntile, s.H, s.Bt), kThreads, smem, st>>>(
        s, ntile, static_cast<const T *>(p.X), static_cast<const T *>(p.B), static_cast<const T *>(p.C), p.cs,
        static_cast<const T *>(p.Hprev), static_cast<float *>(p.Y));
    return launch_end(KK_SSD_OUT, st);
}

cudaError_t launch_ssd_out_simt(const Shape &s, bool bf16, const LayerPtrs &p, cudaStream_t st) {
    return bf16 ? ssd_out_t<__nv_bfloat16>(s, p, st) : ssd_out_t<float>(s, p, st);
}

template <typename T, int KP>
static cudaError_t sma_fwd_kp(const Shape &s, const LayerPtrs &p, cudaStream_t st) {
    constexpr int TT = 16;
    int ntile = (int)((s.S + TT - 1) / TT);
    size_t smem = (2 * TT * s.N + s.N * s.P + s.N) * sizeof(float);
    auto kern = k_sma_fwd_simt<T, KP>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_begin(KK_SMA_FWD, st);
    kern<<<grid3(s.M * ntile, s.H, s.Bt), kThreads, smem, st>>>(s, ntile, p);
    return launch_end(KK_SMA_FWD, st);
}

template <typename T>
static cudaError_t sma_fwd_t(const Shape &s, const LayerPtrs &p, cudaStream_t st) {
    if (s.P <= 32) return sma_fwd_kp<T, 1>(s, p, st);
    if (s.P <= 64) return sma_fwd_kp<T, 2>(s, p, st);
    if (s.P <= 128) return sma_fwd_kp<T, 4>(s, p, st);
    return sma_fwd_kp<T, 8>(s, p, st);
}

cudaError_t launch_sma_fwd_simt(const Shape &s, bool bf16, const LayerPtrs &p, cudaStream_t st) {
    return bf16 ? sma_fwd_t<__nv_bfloat16>(s, p, st) : sma_fwd_t<float>(s, p, st);
}

int decode_splits(int64_t Bt, int64_t H, int64_t n_chunks) {
    const int64_t target = 148 * 64;  // CTAs: several waves of 8 resident CTAs per SM
    int64_t want = (target + Bt * H - 1) / (Bt * H);
    int64_t cap = max((int64_t)1, (n_chunks + 31) / 32);  // keep >= 4 chunks per warp
    return (int)max((int64_t)1, min(want, cap));
}

template <typename T, int VPR>
static cudaError_t decode_vpr(const DecodeArgs &a, cudaStream_t st) {
    int64_t per_split = (a.n_chunks + a.splits - 1) / a.splits;
    if (per_split < 1) per_split = 1;
    size_t smem = (2 * a.N + 2 * (kThreads / 32) + (kThreads / 32) * a.P) * sizeof(float);
    launch_begin(KK_SMA_DECODE, st);
    k_sma_decode<T, VPR><<<grid3(a.splits, a.H, a.Bt), kThreads, smem, st>>>(a, per_split);
    cudaError_t e = launch_end(KK_SMA_DECODE, st);
    if (e != cudaSuccess) return e;
    launch_begin(KK_DECODE_MERGE, st);
    int thr = (int)min((int64_t)kThreads, ((a.P + 31) / 32) * 32);
    k_decode_merge<T><<<(unsigned)(a.Bt * a.H), thr, 0, st>>>(a);
    return launch_end(KK_DECODE_MERGE, st);
}

template <typename T>
static cudaError_t decode_t(const DecodeArgs &a, cudaStream_t st) {
    const int vpr = (int)(a.P * sizeof(T) / 16);
    switch (vpr) {
        case 1: return decode_vpr<T, 1>(a, st);
        case 2: return decode_vpr<T, 2>(a, st);
        case 4: return decode_vpr<T, 4>(a, st);
        case 8: return decode_vpr<T, 8>(a, st);
        case 16: return decode_vpr<T, 16>(a, st);
        case 32: return decode_vpr<T, 32>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_sma_decode(const DecodeArgs &a, bool bf16, cudaStream_t st) {
    return bf16 ? decode_t<__nv_bfloat16>(a, st) : decode_t<float>(a, st);
}

}  // namespace dart

namespace dart {

cudaError_t launch_decode_state(const StateStepArgs &a, bool bf16, cudaStream_t st) {
    launch_begin(KK_DECODE_STATE, st);
    if (bf16)
        k_decode_state<__nv_bfloat16><<<grid3(a.H, a.Bt, 1), kThreads, 0, st>>>(a);
    else
        k_decode_state<float><<<grid3(a.H, a.Bt, 1), kThreads, 0, st>>>(a);
    return launch_end(KK_DECODE_STATE, st);
}

}  // namespace dart
