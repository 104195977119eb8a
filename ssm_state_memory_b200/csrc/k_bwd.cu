// SMA backward on CUDA cores (any supported shape, fp32 or bf16 storage).
//
// State-memory attention (DART §3 eq 8-10) for one token t, head h, with
// k = chunk(t) >= 1 historical chunk memories dH[0..k-1]:
//   V_c = C_t dH[c],  K_c = dH[c] E_t,  l_c = Q_t . K_c / sqrt(N),
//   w = softmax(l) = exp(l - lse_t) (App. C eq 33, 35),  R_t = sum_c w_c V_c.
// Its backward by recomputation (§4 "Efficient Training": the forward keeps only
// R and lse; keys, values, logits and weights are recomputed), for a gradient
// dR_t = dLoss/dR_t:
//   dw_c = dR_t . V_c = C_t . (dH[c] dR_t),  D_t = sum_c w_c dw_c = dR_t . R_t,
//   dl_c = w_c (dw_c - D_t)                          (softmax Jacobian)
//   dQ_t += dl_c K_c / sqrt(N)            dC_t += w_c dH[c] dR_t
//   dE_t += dl_c dH[c]^T Q_t / sqrt(N)    ddH[c] += w_c C_t^T dR_t + dl_c Q_t^T E_t / sqrt(N)
// Q and C are shared by the heads of a group, so dQ and dC sum over the group's heads.
//
// Three kernels: D_t (one warp per token row), the query side (one warp per (token,
// group), looping over the group's heads and the token's history; dQ, dC and dE
// stay in registers), and the memory side (one block per chunk memory, looping over
// every later token; ddH[c] stays in shared memory). Neither needs atomics.
#include <math.h>

#include <algorithm>

#include "dart_internal.cuh"

namespace dart {

namespace {

constexpr int kBwdThreads = 256;

__device__ __forceinline__ float bwd_warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

template <typename T>
__device__ __forceinline__ float ld32(const T *p) {
    return to_f32(p[0]);
}

// D[b, h, t] = dR_t . R_t (rows of P fp32 values); one warp per (b, t, h) row
__global__ void __launch_bounds__(kBwdThreads) k_sma_bwd_delta(Shape s, const float *__restrict__ R,
                                                                const float *__restrict__ dR, float *__restrict__ D) {
    const int lane = threadIdx.x & 31;
    const int64_t rows = s.Bt * s.L * s.H;
    const int64_t wid = ((int64_t)blockIdx.x * kBwdThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kBwdThreads) >> 5;
    for (int64_t r = wid; r < rows; r += nw) {
        const float *a = R + r * s.P, *g = dR + r * s.P;
        float acc = 0.f;
        for (int p = lane; p < s.P; p += 32) acc = fmaf(a[p], g[p], acc);
        acc = bwd_warp_sum(acc);
        if (lane == 0) {
            const int64_t h = r % s.H, bt = r / s.H;  // bt = b * L + t
            const int64_t b = bt / s.L, t = bt % s.L;
            D[(b * s.H + h) * s.L + t] = acc;
        }
    }
}

// Query side: one warp per (b, t, g); NL = ceil(N / 32), PL = ceil(P / 32) values per lane.
// Lane j owns rows n = j + 32 i of the N-vectors (K, K', dQ, dC) and columns p = j + 32 i
// of the P-vectors (dE). Q_t, C_t, E_t and dR_t are staged per warp in shared memory.
template <typename T, int NL, int PL>
__global__ void __launch_bounds__(kBwdThreads) k_sma_bwd_dq_simt(Shape s, BwdArgs a) {
    extern __shared__ float sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = (int)s.N, P = (int)s.P;
    float *q = sm + warp * 2 * (N + P);
    float *cr = q + N, *e = cr + N, *dr = e + P;
    const int64_t item = (int64_t)blockIdx.x * (kBwdThreads / 32) + warp;  // (b, t, g), g fastest
    if (item >= s.Bt * s.L * s.G) return;
    const int64_t g = item % s.G, bt = item / s.G;
    const int64_t b = bt / s.L, t = bt % s.L;
    const int64_t k = t / s.S;
    const int64_t hpg = s.H / s.G;
    const T *Q = static_cast<const T *>(a.Q), *C = static_cast<const T *>(a.C);
    const T *E = static_cast<const T *>(a.E), *dH = static_cast<const T *>(a.dH);
    const float rs = rsqrtf((float)N);
    float dq[NL], dc[NL];
#pragma unroll
    for (int i = 0; i < NL; ++i) dq[i] = dc[i] = 0.f;
    for (int n = lane; n < N; n += 32) {
        q[n] = ld32(Q + (bt * s.G + g) * N + n);
        cr[n] = ld32(C + (bt * s.G + g) * N + n);
    }
    for (int64_t h = g * hpg; h < (g + 1) * hpg; ++h) {
        float de[PL];
#pragma unroll
        for (int i = 0; i < PL; ++i) de[i] = 0.f;
        if (k > 0) {
            __syncwarp();
            for (int p = lane; p < P; p += 32) {
                e[p] = ld32(E + e_row(s, a.EG, bt, h) * P + p);
                dr[p] = a.dR[(bt * s.H + h) * P + p];
            }
            __syncwarp();
            const float lse = a.lse[(b * s.H + h) * s.L + t];
            const float Dt = a.D[(b * s.H + h) * s.L + t];
            for (int64_t c = 0; c < k; ++c) {
                const T *Dm = dH + ((b * s.H + h) * s.M + c) * (int64_t)N * P;
                float kk[NL], kd[NL];
                float lp = 0.f, dwp = 0.f;
#pragma unroll
                for (int i = 0; i < NL; ++i) {
                    const int n = lane + 32 * i;
                    float x = 0.f, y = 0.f;
                    if (n < N) {
                        for (int p = 0; p < P; ++p) {
                            const float v = ld32(Dm + (int64_t)n * P + p);
                            x = fmaf(v, e[p], x);
                            y = fmaf(v, dr[p], y);
                        }
                        lp = fmaf(q[n], x, lp);
                        dwp = fmaf(cr[n], y, dwp);
                    }
                    kk[i] = x;
                    kd[i] = y;
                }
                const float l = bwd_warp_sum(lp) * rs;
                const float dw = bwd_warp_sum(dwp);
                const float w = expf(l - lse);
                const float dl = w * (dw - Dt);
#pragma unroll
                for (int i = 0; i < NL; ++i) {
                    dq[i] = fmaf(dl * rs, kk[i], dq[i]);
                    dc[i] = fmaf(w, kd[i], dc[i]);
                }
#pragma unroll
                for (int i = 0; i < PL; ++i) {
                    const int p = lane + 32 * i;
                    if (p < P) {
                        float u = 0.f;
                        for (int n = 0; n < N; ++n) u = fmaf(ld32(Dm + (int64_t)n * P + p), q[n], u);
                        de[i] = fmaf(dl * rs, u, de[i]);
                    }
                }
            }
        }
        const bool grouped = a.EG > 0 && a.EG != s.H;  // heads of an E group add into its zeroed row
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const int p = lane + 32 * i;
            if (p < P) {
                if (grouped) {
                    if (k > 0) atomicAdd(&a.dE[e_row(s, a.EG, bt, h) * P + p], de[i]);
                } else {
                    a.dE[(bt * s.H + h) * P + p] = de[i];
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NL; ++i) {
        const int n = lane + 32 * i;
        if (n < N) {
            a.dQ[(bt * s.G + g) * N + n] = dq[i];
            a.dC[(bt * s.G + g) * N + n] = dc[i];
        }
    }
}

// Memory side: one block per (c, h, b). ddH[c] (N x P fp32) and dH[c] (fp32) live in shared
// memory; the later tokens go by in batches of TB: their Q, C, E, dR rows are staged, every
// thread forms partial sums of sum_np dH Q E and sum_np dH C dR over its elements, the block
// reduces the 2 TB sums to the logits and dw, and every thread then adds the TB rank-one
// updates to its elements.
constexpr int kTB = 8;

template <typename T>
__global__ void __launch_bounds__(kBwdThreads) k_sma_bwd_ddh_simt(Shape s, BwdArgs a) {
    extern __shared__ float sm[];
    const int N = (int)s.N, P = (int)s.P, NP = N * P;
    const int64_t c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int64_t g = h / (s.H / s.G);
    float *Hs = sm;            // [N][P] dH[c]
    float *G = Hs + NP;        // [N][P] ddH[c] accumulator
    float *qs = G + NP;        // [kTB][N]
    float *cs = qs + kTB * N;  // [kTB][N]
    float *es = cs + kTB * N;  // [kTB][P]
    float *ds = es + kTB * P;  // [kTB][P]
    float *red = ds + kTB * P; // [8 warps][2 kTB] partial sums, then [2 kTB] totals
    float *coef = red + 8 * 2 * kTB + 2 * kTB;  // [2 kTB]: dl/sqrt(N), w per token of the batch
    const T *dH = static_cast<const T *>(a.dH) + ((b * s.H + h) * s.M + c) * (int64_t)NP;
    const T *Q = static_cast<const T *>(a.Q), *C = static_cast<const T *>(a.C), *E = static_cast<const T *>(a.E);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float rs = rsqrtf((float)N);
    for (int i = threadIdx.x; i < NP; i += kBwdThreads) {
        Hs[i] = ld32(dH + i);
        G[i] = 0.f;
    }
    const int64_t t_begin = (c + 1) * s.S;
    for (int64_t t0 = t_begin; t0 < s.L; t0 += kTB) {
        const int tb = (int)min((int64_t)kTB, s.L - t0);
        __syncthreads();  // the previous batch is done with the staging rows
        for (int i = threadIdx.x; i < kTB * N; i += kBwdThreads) {
            const int r = i / N, n = i % N;
            const bool ok = r < tb;
            const int64_t bt = b * s.L + t0 + r;
            qs[i] = ok ? ld32(Q + (bt * s.G + g) * N + n) : 0.f;
            cs[i] = ok ? ld32(C + (bt * s.G + g) * N + n) : 0.f;
        }
        for (int i = threadIdx.x; i < kTB * P; i += kBwdThreads) {
            const int r = i / P, p = i % P;
            const bool ok = r < tb;
            const int64_t bt = b * s.L + t0 + r;
            es[i] = ok ? ld32(E + e_row(s, a.EG, bt, h) * P + p) : 0.f;
            ds[i] = ok ? a.dR[(bt * s.H + h) * P + p] : 0.f;
        }
        __syncthreads();
        float part[2 * kTB];
#pragma unroll
        for (int r = 0; r < 2 * kTB; ++r) part[r] = 0.f;
        for (int i = threadIdx.x; i < NP; i += kBwdThreads) {
            const int n = i / P, p = i % P;
            const float v = Hs[i];
#pragma unroll
            for (int r = 0; r < kTB; ++r) {
                part[r] = fmaf(v * qs[r * N + n], es[r * P + p], part[r]);
                part[kTB + r] = fmaf(v * cs[r * N + n], ds[r * P + p], part[kTB + r]);
            }
        }
#pragma unroll
        for (int r = 0; r < 2 * kTB; ++r) {
            const float v = bwd_warp_sum(part[r]);
            if (lane == 0) red[warp * 2 * kTB + r] = v;
        }
        __syncthreads();
        if (threadIdx.x < kTB) {
            const int r = threadIdx.x;
            float l = 0.f, dw = 0.f;
            for (int w8 = 0; w8 < kBwdThreads / 32; ++w8) {
                l += red[w8 * 2 * kTB + r];
                dw += red[w8 * 2 * kTB + kTB + r];
            }
            float cl = 0.f, cw = 0.f;
            if (r < tb) {
                const int64_t t = t0 + r;
                const float w = expf(l * rs - a.lse[(b * s.H + h) * s.L + t]);
                cl = w * (dw - a.D[(b * s.H + h) * s.L + t]) * rs;
                cw = w;
            }
            coef[r] = cl;
            coef[kTB + r] = cw;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < NP; i += kBwdThreads) {
            const int n = i / P, p = i % P;
            float acc = G[i];
#pragma unroll
            for (int r = 0; r < kTB; ++r) {
                acc = fmaf(coef[r] * qs[r * N + n], es[r * P + p], acc);
                acc = fmaf(coef[kTB + r] * cs[r * N + n], ds[r * P + p], acc);
            }
            G[i] = acc;
        }
    }
    __syncthreads();
    float *out = a.ddH + ((b * s.H + h) * s.M + c) * (int64_t)NP;
    for (int i = threadIdx.x; i < NP; i += kBwdThreads) out[i] = G[i];
}

// ---------------------------------------------------------------------------
// Normalised score branch (App. B.1 eq 25-27). Forward: Qb = iq Q_t, Eb = ie E_t (RMSNorm, unit
// weight), r_{c,n} = (mean_p dH[c]_{n,p}^2 + eps)^(-1/2), K_c = r_c (.) (dH[c] Eb), l_c = Qb . K_c / sqrt(N),
// values as in the plain branch. With a_c = w_c (dw_c - D_t) / sqrt(N):
//   dQb = sum_c a_c K_c,  dEb = sum_c a_c dH[c]^T (r_c (.) Qb),  dC_t = sum_c w_c dH[c] dR_t,
//   ddH[c]_{n,p} = sum_t w_c C_n dR_p + a_c Qb_n (r_n Eb_p - r_n^3 (dH[c] Eb)_n dH[c]_{n,p} / P),
//   dQ_t = iq dQb - iq^3 Q_t (Q_t . dQb) / N,  dE_t = ie dEb - ie^3 E_t (E_t . dEb) / P.
// ---------------------------------------------------------------------------

// Query side: one warp per (b, t, g); lane j owns rows n = j + 32 i and columns p = j + 32 i.
template <typename T, int NL, int PL>
__global__ void __launch_bounds__(kBwdThreads) k_sma_bwd_dq_norm_simt(Shape s, BwdArgs a, float eps) {
    extern __shared__ float sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = (int)s.N, P = (int)s.P;
    float *q = sm + warp * (4 * N + 3 * P);
    float *cr = q + N, *qb = cr + N, *rr = qb + N, *e = rr + N, *eb = e + P, *dr = eb + P;
    const int64_t item = (int64_t)blockIdx.x * (kBwdThreads / 32) + warp;  // (b, t, g), g fastest
    if (item >= s.Bt * s.L * s.G) return;
    const int64_t g = item % s.G, bt = item / s.G;
    const int64_t b = bt / s.L, t = bt % s.L;
    const int64_t k = t / s.S;
    const int64_t hpg = s.H / s.G;
    const T *Q = static_cast<const T *>(a.Q), *C = static_cast<const T *>(a.C);
    const T *E = static_cast<const T *>(a.E), *dH = static_cast<const T *>(a.dH);
    const float rs = rsqrtf((float)N);
    float sq = 0.f;
    for (int n = lane; n < N; n += 32) {
        q[n] = ld32(Q + (bt * s.G + g) * N + n);
        cr[n] = ld32(C + (bt * s.G + g) * N + n);
        sq = fmaf(q[n], q[n], sq);
    }
    const float iq = rsqrtf(bwd_warp_sum(sq) / (float)N + eps);
    for (int n = lane; n < N; n += 32) qb[n] = q[n] * iq;
    float dqb[NL], dc[NL];
#pragma unroll
    for (int i = 0; i < NL; ++i) dqb[i] = dc[i] = 0.f;
    for (int64_t h = g * hpg; h < (g + 1) * hpg; ++h) {
        float de[PL];
#pragma unroll
        for (int i = 0; i < PL; ++i) de[i] = 0.f;
        if (k > 0) {
            __syncwarp();
            float se = 0.f;
            for (int p = lane; p < P; p += 32) {
                e[p] = ld32(E + (bt * s.H + h) * P + p);
                dr[p] = a.dR[(bt * s.H + h) * P + p];
                se = fmaf(e[p], e[p], se);
            }
            const float ie = rsqrtf(bwd_warp_sum(se) / (float)P + eps);
            for (int p = lane; p < P; p += 32) eb[p] = e[p] * ie;
            __syncwarp();
            // pass 1: the softmax statistics of this token from the recomputed logits (online, App. C eq
            // 28-31): lse, and D = sum_c w_c dw_c; written for the memory-side kernel
            float lse, Dt;
            {
                float m = -INFINITY, den = 0.f, sdw = 0.f;
                for (int64_t c = 0; c < k; ++c) {
                    const T *Dm = dH + ((b * s.H + h) * s.M + c) * (int64_t)N * P;
                    float lp = 0.f, dwp = 0.f;
#pragma unroll
                    for (int i = 0; i < NL; ++i) {
                        const int n = lane + 32 * i;
                        if (n < N) {
                            float x = 0.f, y = 0.f, z = 0.f;
                            for (int p = 0; p < P; ++p) {
                                const float v = ld32(Dm + (int64_t)n * P + p);
                                x = fmaf(v, eb[p], x);
                                y = fmaf(v, dr[p], y);
                                z = fmaf(v, v, z);
                            }
                            lp = fmaf(qb[n], x * rsqrtf(z / (float)P + eps), lp);
                            dwp = fmaf(cr[n], y, dwp);
                        }
                    }
                    const float l = bwd_warp_sum(lp) * rs;
                    const float dw = bwd_warp_sum(dwp);
                    const float mn = fmaxf(m, l);
                    const float f = expf(m - mn), wl = expf(l - mn);
                    den = den * f + wl;
                    sdw = sdw * f + wl * dw;
                    m = mn;
                }
                lse = m + logf(den);
                Dt = sdw / den;
                if (lane == 0) {
                    a.D[(b * s.H + h) * s.L + t] = Dt;
                    a.lse_rc[(b * s.H + h) * s.L + t] = lse;
                }
            }
            float deb[PL];
#pragma unroll
            for (int i = 0; i < PL; ++i) deb[i] = 0.f;
            for (int64_t c = 0; c < k; ++c) {
                const T *Dm = dH + ((b * s.H + h) * s.M + c) * (int64_t)N * P;
                float kk[NL], kd[NL];
                float lp = 0.f, dwp = 0.f;
#pragma unroll
                for (int i = 0; i < NL; ++i) {
                    const int n = lane + 32 * i;
                    float x = 0.f, y = 0.f, z = 0.f;
                    if (n < N) {
                        for (int p = 0; p < P; ++p) {
                            const float v = ld32(Dm + (int64_t)n * P + p);
                            x = fmaf(v, eb[p], x);
                            y = fmaf(v, dr[p], y);
                            z = fmaf(v, v, z);
                        }
                        const float r = rsqrtf(z / (float)P + eps);
                        rr[n] = r;
                        x *= r;  // K_n = r_n (dH Eb)_n
                        lp = fmaf(qb[n], x, lp);
                        dwp = fmaf(cr[n], y, dwp);
                    }
                    kk[i] = x;
                    kd[i] = y;
                }
                const float l = bwd_warp_sum(lp) * rs;
                const float dw = bwd_warp_sum(dwp);
                const float w = expf(l - lse);
                const float aa = w * (dw - Dt) * rs;
#pragma unroll
                for (int i = 0; i < NL; ++i) {
                    dqb[i] = fmaf(aa, kk[i], dqb[i]);
                    dc[i] = fmaf(w, kd[i], dc[i]);
                }
                __syncwarp();  // rr of this chunk
#pragma unroll
                for (int i = 0; i < PL; ++i) {
                    const int p = lane + 32 * i;
                    if (p < P) {
                        float u = 0.f;
                        for (int n = 0; n < N; ++n) u = fmaf(ld32(Dm + (int64_t)n * P + p), rr[n] * qb[n], u);
                        deb[i] = fmaf(aa, u, deb[i]);
                    }
                }
                __syncwarp();  // rr is rewritten by the next chunk
            }
            // through RMSNorm(E_t)
            float ed = 0.f;
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int p = lane + 32 * i;
                if (p < P) ed = fmaf(e[p], deb[i], ed);
            }
            ed = bwd_warp_sum(ed);
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int p = lane + 32 * i;
                if (p < P) de[i] = ie * deb[i] - ie * ie * ie * e[p] * ed / (float)P;
            }
        }
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const int p = lane + 32 * i;
            if (p < P) a.dE[(bt * s.H + h) * P + p] = de[i];
        }
    }
    // through RMSNorm(Q_t)
    float qd = 0.f;
#pragma unroll
    for (int i = 0; i < NL; ++i) {
        const int n = lane + 32 * i;
        if (n < N) qd = fmaf(q[n], dqb[i], qd);
    }
    qd = bwd_warp_sum(qd);
#pragma unroll
    for (int i = 0; i < NL; ++i) {
        const int n = lane + 32 * i;
        if (n < N) {
            a.dQ[(bt * s.G + g) * N + n] = iq * dqb[i] - iq * iq * iq * q[n] * qd / (float)N;
            a.dC[(bt * s.G + g) * N + n] = dc[i];
        }
    }
}

// Memory side: one block per (c, h, b), dH[c] and its ddH accumulator in shared memory, the later
// tokens in batches of kTB = 8 (one warp per token for the per-token reductions).
template <typename T>
__global__ void __launch_bounds__(kBwdThreads) k_sma_bwd_ddh_norm_simt(Shape s, BwdArgs a, float eps) {
    extern __shared__ float sm[];
    const int N = (int)s.N, P = (int)s.P, NP = N * P;
    const int64_t c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int64_t g = h / (s.H / s.G);
    float *Hs = sm;              // [N][P]
    float *Gm = Hs + NP;         // [N][P] accumulator
    float *rr = Gm + NP;         // [N]
    float *qs = rr + N;          // [kTB][N] Qb
    float *cs = qs + kTB * N;    // [kTB][N] C
    float *kv = cs + kTB * N;    // [kTB][N] (dH Eb)_n
    float *kd = kv + kTB * N;    // [kTB][N] (dH dR)_n
    float *es = kd + kTB * N;    // [kTB][P] Eb
    float *ds = es + kTB * P;    // [kTB][P] dR
    float *coef = ds + kTB * P;  // [2 kTB]: w, a per token of the batch
    const T *dH = static_cast<const T *>(a.dH) + ((b * s.H + h) * s.M + c) * (int64_t)NP;
    const T *Q = static_cast<const T *>(a.Q), *C = static_cast<const T *>(a.C), *E = static_cast<const T *>(a.E);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float rs = rsqrtf((float)N);
    for (int i = threadIdx.x; i < NP; i += kBwdThreads) {
        Hs[i] = ld32(dH + i);
        Gm[i] = 0.f;
    }
    __syncthreads();
    for (int n = threadIdx.x; n < N; n += kBwdThreads) {
        float z = 0.f;
        for (int p = 0; p < P; ++p) z = fmaf(Hs[n * P + p], Hs[n * P + p], z);
        rr[n] = rsqrtf(z / (float)P + eps);
    }
    for (int64_t t0 = (c + 1) * s.S; t0 < s.L; t0 += kTB) {
        const int tb = (int)min((int64_t)kTB, s.L - t0);
        __syncthreads();  // the previous batch is done with the staged rows
        {  // warp r stages token r: Qb, C, Eb, dR
            const int r = warp;
            const bool ok = r < tb;
            const int64_t bt = b * s.L + t0 + r;
            float sq = 0.f, se = 0.f;
            for (int n = lane; n < N; n += 32) {
                const float v = ok ? ld32(Q + (bt * s.G + g) * N + n) : 0.f;
                qs[r * N + n] = v;
                cs[r * N + n] = ok ? ld32(C + (bt * s.G + g) * N + n) : 0.f;
                sq = fmaf(v, v, sq);
            }
            for (int p = lane; p < P; p += 32) {
                const float v = ok ? ld32(E + (bt * s.H + h) * P + p) : 0.f;
                es[r * P + p] = v;
                ds[r * P + p] = ok ? a.dR[(bt * s.H + h) * P + p] : 0.f;
                se = fmaf(v, v, se);
            }
            const float iq = rsqrtf(bwd_warp_sum(sq) / (float)N + eps);
            const float ie = rsqrtf(bwd_warp_sum(se) / (float)P + eps);
            __syncwarp();
            for (int n = lane; n < N; n += 32) qs[r * N + n] *= iq;
            for (int p = lane; p < P; p += 32) es[r * P + p] *= ie;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < kTB * N; i += kBwdThreads) {  // (dH Eb)_n and (dH dR)_n per token
            const int r = i / N, n = i % N;
            float x = 0.f, y = 0.f;
            for (int p = 0; p < P; ++p) {
                const float v = Hs[n * P + p];
                x = fmaf(v, es[r * P + p], x);
                y = fmaf(v, ds[r * P + p], y);
            }
            kv[i] = x;
            kd[i] = y;
        }
        __syncthreads();
        {  // warp r: the logit, w and a of token r
            const int r = warp;
            float lp = 0.f, dwp = 0.f;
            for (int n = lane; n < N; n += 32) {
                lp = fmaf(qs[r * N + n] * rr[n], kv[r * N + n], lp);
                dwp = fmaf(cs[r * N + n], kd[r * N + n], dwp);
            }
            lp = bwd_warp_sum(lp);
            dwp = bwd_warp_sum(dwp);
            if (lane == 0) {
                float w = 0.f, aa = 0.f;
                if (r < tb) {
                    const int64_t t = t0 + r;
                    w = expf(lp * rs - a.lse[(b * s.H + h) * s.L + t]);
                    aa = w * (dwp - a.D[(b * s.H + h) * s.L + t]) * rs;
                }
                coef[r] = w;
                coef[kTB + r] = aa;
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < NP; i += kBwdThreads) {
            const int n = i / P, p = i % P;
            const float r = rr[n], r3 = r * r * r * Hs[i] / (float)P;
            float acc = Gm[i];
#pragma unroll
            for (int q = 0; q < kTB; ++q) {
                acc = fmaf(coef[q] * cs[q * N + n], ds[q * P + p], acc);
                acc = fmaf(coef[kTB + q] * qs[q * N + n], r * es[q * P + p] - r3 * kv[q * N + n], acc);
            }
            Gm[i] = acc;
        }
    }
    __syncthreads();
    float *out = a.ddH + ((b * s.H + h) * s.M + c) * (int64_t)NP;
    for (int i = threadIdx.x; i < NP; i += kBwdThreads) out[i] = Gm[i];
}

template <typename T, int NL, int PL>
void launch_dq_norm(const Shape &s, const BwdArgs &a, float eps, cudaStream_t st) {
    const size_t smem = (size_t)(kBwdThreads / 32) * (4 * s.N + 3 * s.P) * sizeof(float);
    const int64_t items = s.Bt * s.L * s.G;
    const int64_t blocks = (items + kBwdThreads / 32 - 1) / (kBwdThreads / 32);
    k_sma_bwd_dq_norm_simt<T, NL, PL><<<(unsigned)blocks, kBwdThreads, smem, st>>>(s, a, eps);
}

template <typename T, int NL>
void launch_dq_norm_p(const Shape &s, const BwdArgs &a, float eps, cudaStream_t st) {
    switch ((int)((s.P + 31) / 32)) {
        case 1: launch_dq_norm<T, NL, 1>(s, a, eps, st); break;
        case 2: launch_dq_norm<T, NL, 2>(s, a, eps, st); break;
        case 3: case 4: launch_dq_norm<T, NL, 4>(s, a, eps, st); break;
        default: launch_dq_norm<T, NL, 8>(s, a, eps, st); break;
    }
}

template <typename T>
void launch_dq_norm_n(const Shape &s, const BwdArgs &a, float eps, cudaStream_t st) {
    switch ((int)((s.N + 31) / 32)) {
        case 1: launch_dq_norm_p<T, 1>(s, a, eps, st); break;
        case 2: launch_dq_norm_p<T, 2>(s, a, eps, st); break;
        case 3: case 4: launch_dq_norm_p<T, 4>(s, a, eps, st); break;
        default: launch_dq_norm_p<T, 8>(s, a, eps, st); break;
    }
}

size_t ddh_norm_smem(const Shape &s) {
    return (size_t)(2 * s.N * s.P + s.N + 4 * kTB * s.N + 2 * kTB * s.P + 2 * kTB) * sizeof(float);
}

template <typename T, int NL, int PL>
cudaError_t launch_dq(const Shape &s, const BwdArgs &a, cudaStream_t st) {
    const size_t smem = (size_t)(kBwdThreads / 32) * 2 * (s.N + s.P) * sizeof(float);
    const int64_t items = s.Bt * s.L * s.G;
    const int64_t blocks = (items + kBwdThreads / 32 - 1) / (kBwdThreads / 32);
    k_sma_bwd_dq_simt<T, NL, PL><<<(unsigned)blocks, kBwdThreads, smem, st>>>(s, a);
    return cudaSuccess;  // launch errors are picked up by launch_end
}

template <typename T, int NL>
cudaError_t launch_dq_p(const Shape &s, const BwdArgs &a, cudaStream_t st) {
    const int pl = (int)((s.P + 31) / 32);
    switch (pl) {
        case 1: return launch_dq<T, NL, 1>(s, a, st);
        case 2: return launch_dq<T, NL, 2>(s, a, st);
        case 3: case 4: return launch_dq<T, NL, 4>(s, a, st);
        default: return launch_dq<T, NL, 8>(s, a, st);
    }
}

template <typename T>
cudaError_t launch_dq_n(const Shape &s, const BwdArgs &a, cudaStream_t st) {
    const int nl = (int)((s.N + 31) / 32);
    switch (nl) {
        case 1: return launch_dq_p<T, 1>(s, a, st);
        case 2: return launch_dq_p<T, 2>(s, a, st);
        case 3: case 4: return launch_dq_p<T, 4>(s, a, st);
        default: return launch_dq_p<T, 8>(s, a, st);
    }
}

size_t ddh_smem(const Shape &s) {
    return (size_t)(2 * s.N * s.P + 2 * kTB * s.N + 2 * kTB * s.P + 8 * 2 * kTB + 2 * kTB + 2 * kTB) * sizeof(float);
}

template <typename T>
cudaError_t ddh_attr(const Shape &s) {
    return cudaFuncSetAttribute(k_sma_bwd_ddh_simt<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ddh_smem(s));
}

template <typename T>
void launch_ddh(const Shape &s, const BwdArgs &a, cudaStream_t st) {
    k_sma_bwd_ddh_simt<T><<<dim3((unsigned)s.M, (unsigned)s.H, (unsigned)s.Bt), kBwdThreads, ddh_smem(s), st>>>(s, a);
}

}  // namespace

cudaError_t launch_sma_bwd_delta(const Shape &s, const BwdArgs &a, cudaStream_t st) {
    const int64_t rows = s.Bt * s.L * s.H;
    const int64_t blocks = std::min<int64_t>((rows + kBwdThreads / 32 - 1) / (kBwdThreads / 32), 148 * 16);
    launch_begin(KK_SMA_BWD_DELTA, st);
    k_sma_bwd_delta<<<(unsigned)blocks, kBwdThreads, 0, st>>>(s, a.R, a.dR, a.D);
    return launch_end(KK_SMA_BWD_DELTA, st);
}

cudaError_t launch_sma_bwd_norm_simt(const Shape &s, bool bf16, const BwdArgs &a, float eps, cudaStream_t st) {
    const size_t smem = ddh_norm_smem(s);
    cudaError_t e = bf16 ? cudaFuncSetAttribute(k_sma_bwd_ddh_norm_simt<__nv_bfloat16>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                         : cudaFuncSetAttribute(k_sma_bwd_ddh_norm_simt<float>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
        set_last_error("cudaFuncSetAttribute(sma_bwd_ddh_norm)", e);
        return e;
    }
    launch_begin(KK_SMA_BWD_DQ, st);
    if (bf16)
        launch_dq_norm_n<__nv_bfloat16>(s, a, eps, st);
    else
        launch_dq_norm_n<float>(s, a, eps, st);
    e = launch_end(KK_SMA_BWD_DQ, st);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)s.M, (unsigned)s.H, (unsigned)s.Bt);
    launch_begin(KK_SMA_BWD_DDH, st);
    if (bf16)
        k_sma_bwd_ddh_norm_simt<__nv_bfloat16><<<grid, kBwdThreads, smem, st>>>(s, a, eps);
    else
        k_sma_bwd_ddh_norm_simt<float><<<grid, kBwdThreads, smem, st>>>(s, a, eps);
    return launch_end(KK_SMA_BWD_DDH, st);
}

cudaError_t launch_sma_bwd_simt(const Shape &s, bool bf16, const BwdArgs &a, cudaStream_t st) {
    cudaError_t e = bf16 ? ddh_attr<__nv_bfloat16>(s) : ddh_attr<float>(s);
    if (e != cudaSuccess) {
        set_last_error("cudaFuncSetAttribute(sma_bwd_ddh)", e);
        return e;
    }
    if (a.EG > 0 && a.EG != s.H) {  // grouped E: the heads of a group add their dE into a zeroed row
        e = cudaMemsetAsync(a.dE, 0, (size_t)(s.Bt * s.L * a.EG * s.P) * sizeof(float), st);
        if (e != cudaSuccess) {
            set_last_error("cudaMemsetAsync(dE)", e);
            return e;
        }
    }
    launch_begin(KK_SMA_BWD_DQ, st);
    if (bf16)
        launch_dq_n<__nv_bfloat16>(s, a, st);
    else
        launch_dq_n<float>(s, a, st);
    e = launch_end(KK_SMA_BWD_DQ, st);
    if (e != cudaSuccess) return e;
    launch_begin(KK_SMA_BWD_DDH, st);
    if (bf16)
        launch_ddh<__nv_bfloat16>(s, a, st);
    else
        launch_ddh<float>(s, a, st);
    return launch_end(KK_SMA_BWD_DDH, st);
}

}  // namespace dart
