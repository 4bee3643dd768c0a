// simt.cuh -- general CUDA-core kernels for every TTT path and both storage types.
//
// These serve the fp32 inputs (whose 1e-4 accuracy bar rules out bf16 tensor cores) and any
// shape the tensor-core kernels do not cover.  One thread owns one output value and sums in
// fp32 over the reduction axis, so the code follows the definition step by step:
//   full-batch step  W* = W0 - eta * grad l(W0),  l(W) = (1/N) sum_i 1/2 ||F_W(k_i) - v_i||^2,
//   then o_i = F_{W*}(q_i)  ("ViT^3" blog: attention rewritten as online learning, steps 1-3;
//   single epoch, full batch, lr 1.0 per its inner-training study).
// Every intermediate lives in the caller's workspace (fp32); the long sums over tokens are
// accumulated in fp64, because the step W0 - eta*grad can cancel most of W0 (the 3x3 conv
// model at eta = 1 keeps about 2% of it), which magnifies summation error in W*.
#pragma once
#include "common.cuh"

namespace simt {

constexpr int TPB = 256;

// ------------------------------------------------------------------ TTT-Linear -------
// gc[u][i][c] = sum_t k[u][t][i] * X[u][t][c'],  X = K for c < d, V for c >= d (c' = c mod d)
template <typename T>
__global__ void __launch_bounds__(TPB) linear_gram(const T* __restrict__ k, const T* __restrict__ v,
                                                   float* __restrict__ gc, int N, int d) {
    const long long u = blockIdx.x;
    const int e = blockIdx.y * TPB + threadIdx.x;
    const int w2 = 2 * d;
    if (e >= d * w2) return;
    const int i = e / w2, c = e % w2;
    const T* ku = k + u * N * d;
    const T* xu = (c < d ? k : v) + u * N * d;
    const int cc = c < d ? c : c - d;
    double acc = 0.0;
    for (int t = 0; t < N; ++t) acc = fma((double)to_f(ku[(long long)t * d + i]), (double)to_f(xu[(long long)t * d + cc]), acc);
    gc[u * d * w2 + e] = (float)acc;
}

// W*[u] = W0[h] - (eta/N) (G W0[h] - C)
__global__ void __launch_bounds__(TPB) linear_update(const float* __restrict__ gc, const float* __restrict__ w0,
                                                     float* __restrict__ wst, float* __restrict__ w_star_out,
                                                     int H, int d, float eta_over_n) {
    const long long u = blockIdx.x;
    const int e = blockIdx.y * TPB + threadIdx.x;
    if (e >= d * d) return;
    const int i = e / d, j = e % d;
    const float* G = gc + u * 2 * d * d + (long long)i * 2 * d;  // row i of [G | C]
    const float* W0 = w0 + (u % H) * d * d;
    float s = 0.f;
    for (int m = 0; m < d; ++m) s = fmaf(G[m], W0[m * d + j], s);
    const float w = W0[e] - eta_over_n * (s - G[d + j]);
    wst[u * d * d + e] = w;
    if (w_star_out) w_star_out[u * d * d + e] = w;
}

// out[u][t][j] = sum_m x[u][t][m] * W[u][m][j]
template <typename T>
__global__ void __launch_bounds__(TPB) linear_apply(const T* __restrict__ x, const float* __restrict__ w,
                                                    T* __restrict__ out, int N, int d) {
    const long long u = blockIdx.x;
    const long long e = (long long)blockIdx.y * TPB + threadIdx.x;
    if (e >= (long long)N * d) return;
    const long long t = e / d;
    const int j = (int)(e % d);
    const float* W = w + u * d * d;
    const T* xt = x + u * N * d + t * d;
    float s = 0.f;
    for (int m = 0; m < d; ++m) s = fmaf(to_f(xt[m]), W[m * d + j], s);
    out[u * N * d + e] = from_f<T>(s);
}

// ------------------------------------------------------------------ 3x3 depthwise conv -
// channels-last [B][Hg][Wg][C]; taps [C][3][3] (per image when per_image != 0: [B][C][3][3])
template <typename T>
__device__ __forceinline__ float dw_tap_sum(const T* img, const float* wc, int Hg, int Wg, int C, int y,
                                            int x, int c) {
    float s = 0.f;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        const int yy = y + a - 1;
        if (yy < 0 || yy >= Hg) continue;
#pragma unroll
        for (int b = 0; b < 3; ++b) {
            const int xx = x + b - 1;
            if (xx < 0 || xx >= Wg) continue;
            s = fmaf(wc[a * 3 + b], to_f(img[((long long)yy * Wg + xx) * C + c]), s);
        }
    }
    return s;
}

// r[b][p][c] = conv_{w0}(K)(p, c) - V(p, c)
template <typename T>
__global__ void __launch_bounds__(TPB) dwconv_residual(const T* __restrict__ k, const T* __restrict__ v,
                                                       const float* __restrict__ w0, float* __restrict__ r,
                                                       int Hg, int Wg, int C) {
    const long long b = blockIdx.x;
    const long long e = (long long)blockIdx.y * TPB + threadIdx.x;
    const long long NC = (long long)Hg * Wg * C;
    if (e >= NC) return;
    const int c = (int)(e % C);
    const long long p = e / C;
    const int y = (int)(p / Wg), x = (int)(p % Wg);
    r[b * NC + e] = dw_tap_sum(k + b * NC, w0 + c * 9, Hg, Wg, C, y, x, c) - to_f(v[b * NC + e]);
}

// w*[b][c][tap] = w0[c][tap] - (eta/N) sum_p r(p, c) K(p + offset(tap), c)
template <typename T>
__global__ void __launch_bounds__(TPB) dwconv_update(const T* __restrict__ k, const float* __restrict__ r,
                                                     const float* __restrict__ w0, float* __restrict__ wst,
                                                     float* __restrict__ w_star_out, int Hg, int Wg, int C,
                                                     float eta_over_n) {
    const long long b = blockIdx.x;
    const int e = blockIdx.y * TPB + threadIdx.x;
    if (e >= 9 * C) return;
    const int tap = e / C, c = e % C;
    const int da = tap / 3 - 1, db = tap % 3 - 1;
    const long long NC = (long long)Hg * Wg * C;
    const T* kb = k + b * NC;
    const float* rb = r + b * NC;
    double acc = 0.0;
    for (int y = 0; y < Hg; ++y) {
        const int yy = y + da;
        if (yy < 0 || yy >= Hg) continue;
        for (int x = 0; x < Wg; ++x) {
            const int xx = x + db;
            if (xx < 0 || xx >= Wg) continue;
            acc = fma((double)rb[((long long)y * Wg + x) * C + c], (double)to_f(kb[((long long)yy * Wg + xx) * C + c]), acc);
        }
    }
    const float w = (float)((double)w0[c * 9 + tap] - (double)eta_over_n * acc);
    wst[(b * C + c) * 9 + tap] = w;
    if (w_star_out) w_star_out[(b * C + c) * 9 + tap] = w;
}

template <typename T>
__global__ void __launch_bounds__(TPB) dwconv_apply(const T* __restrict__ q, const float* __restrict__ wst,
                                                    T* __restrict__ out, int Hg, int Wg, int C) {
    const long long b = blockIdx.x;
    const long long e = (long long)blockIdx.y * TPB + threadIdx.x;
    const long long NC = (long long)Hg * Wg * C;
    if (e >= NC) return;
    const int c = (int)(e % C);
    const long long p = e / C;
    const int y = (int)(p / Wg), x = (int)(p % Wg);
    out[b * NC + e] = from_f<T>(dw_tap_sum(q + b * NC, wst + (b * C + c) * 9, Hg, Wg, C, y, x, c));
}

// ------------------------------------------------------------------ TTT-MLP ----------
// a[u][t][m] = gelu(sum_i x[u][t][i] W1[i][m]); gp = gelu'(...) when gp != nullptr.
// W1 is per head ([H][d][hd]) or per unit ([U][d][hd]) when per_unit != 0.
template <typename T>
__global__ void __launch_bounds__(TPB) mlp_hidden(const T* __restrict__ x, const float* __restrict__ w1,
                                                  float* __restrict__ a, float* __restrict__ gp, int H, int N,
                                                  int d, int hd, int per_unit) {
    const long long u = blockIdx.x;
    const long long e = (long long)blockIdx.y * TPB + threadIdx.x;
    if (e >= (long long)N * hd) return;
    const long long t = e / hd;
    const int m = (int)(e % hd);
    const float* W1 = w1 + (per_unit ? u : u % H) * d * hd;
    const T* xt = x + u * N * d + t * d;
    float z = 0.f;
    for (int i = 0; i < d; ++i) z = fmaf(to_f(xt[i]), W1[i * hd + m], z);
    float g;
    a[u * N * hd + e] = gelu_tanh_f(z, gp ? &g : nullptr);
    if (gp) gp[u * N * hd + e] = g;
}

// y[u][t][j] = sum_m a[u][t][m] W2[m][j]; APPLY: out = y, else r = y - v
template <typename T, bool APPLY>
__global__ void __launch_bounds__(TPB) mlp_out(const float* __restrict__ a, const float* __restrict__ w2,
                                               const T* __restrict__ v, float* __restrict__ r, T* __restrict__ out,
                                               int H, int N, int d, int hd, int per_unit) {
    const long long u = blockIdx.x;
    const long long e = (long long)blockIdx.y * TPB + threadIdx.x;
    if (e >= (long long)N * d) return;
    const long long t = e / d;
    const int j = (int)(e % d);
    const float* W2 = w2 + (per_unit ? u : u % H) * hd * d;
    const float* at = a + u * N * hd + t * hd;
    float s = 0.f;
    for (int m = 0; m < hd; ++m) s = fmaf(at[m], W2[m * d + j], s);
    if (APPLY)
        out[u * N * d + e] = from_f<T>(s);
    else
        r[u * N * d + e] = s - to_f(v[u * N * d + e]);
}

// dz[u][t][m] = gelu'(z) * sum_j r[u][t][j] W2[h][m][j]   (written over gp)
__global__ void __launch_bounds__(TPB) mlp_dz(const float* __restrict__ r, const float* __restrict__ w2,
                                              float* __restrict__ gp_dz, int H, int N, int d, int hd) {
    const long long u = blockIdx.x;
    const long long e = (long long)blockIdx.y * TPB + threadIdx.x;
    if (e >= (long long)N * hd) return;
    const long long t = e / hd;
    const int m = (int)(e % hd);
    const float* W2 = w2 + (u % H) * hd * d + (long long)m * d;
    const float* rt = r + u * N * d + t * d;
    float s = 0.f;
    for (int j = 0; j < d; ++j) s = fmaf(rt[j], W2[j], s);
    gp_dz[u * N * hd + e] *= s;
}

// W1*[u][i][m] = W1[h][i][m] - (eta/N) sum_t k[t][i] dz[t][m]
template <typename T>
__global__ void __launch_bounds__(TPB) mlp_update_w1(const T* __restrict__ k, const float* __restrict__ dz,
                                                     const float* __restrict__ w1, float* __restrict__ w1s,
                                                     float* __restrict__ w1_out, int H, int N, int d, int hd,
                                                     float eta_over_n) {
    const long long u = blockIdx.x;
    const int e = blockIdx.y * TPB + threadIdx.x;
    if (e >= d * hd) return;
    const int i = e / hd, m = e % hd;
    const T* ku = k + u * N * d;
    const float* du = dz + u * N * hd;
    double s = 0.0;
    for (int t = 0; t < N; ++t) s = fma((double)to_f(ku[(long long)t * d + i]), (double)du[(long long)t * hd + m], s);
    const float w = (float)((double)w1[(u % H) * d * hd + e] - (double)eta_over_n * s);
    w1s[u * d * hd + e] = w;
    if (w1_out) w1_out[u * d * hd + e] = w;
}

// W2*[u][m][j] = W2[h][m][j] - (eta/N) sum_t a[t][m] r[t][j]
__global__ void __launch_bounds__(TPB) mlp_update_w2(const float* __restrict__ a, const float* __restrict__ r,
                                                     const float* __restrict__ w2, float* __restrict__ w2s,
                                                     float* __restrict__ w2_out, int H, int N, int d, int hd,
                                                     float eta_over_n) {
    const long long u = blockIdx.x;
    const int e = blockIdx.y * TPB + threadIdx.x;
    if (e >= hd * d) return;
    const int m = e / d, j = e % d;
    const float* au = a + u * N * hd;
    const float* ru = r + u * N * d;
    double s = 0.0;
    for (int t = 0; t < N; ++t) s = fma((double)au[(long long)t * hd + m], (double)ru[(long long)t * d + j], s);
    const float w = (float)((double)w2[(u % H) * hd * d + e] - (double)eta_over_n * s);
    w2s[u * hd * d + e] = w;
    if (w2_out) w2_out[u * hd * d + e] = w;
}

// ------------------------------------------------------------------ chunked scan -----
// One block per (unit, direction).  Shared memory: W [d][d], G [d][d], R [RB][d] (fp32).
// Direction 0 visits chunks 0..nc-1, direction 1 visits them nc-1..0 (reverse raster);
// the order of tokens inside a chunk does not change its sums.  The grid's y extent is the
// number of directions run (1 or 2), the first of them is dir0; each writes its own partial.
constexpr int CH_RB = 32;

template <typename T>
__global__ void __launch_bounds__(TPB) chunked_scan(const T* __restrict__ q, const T* __restrict__ k,
                                                    const T* __restrict__ v, const float* __restrict__ w0,
                                                    float* __restrict__ opart, int H, int N, int d, int chunk,
                                                    float eta_over_b, int dir0) {
    extern __shared__ float sm[];
    float* W = sm;
    float* G = W + d * d;
    float* R = G + d * d;
    const long long u = blockIdx.x;
    const int dir = dir0 + (int)blockIdx.y;
    const int dd = d * d;
    const long long base = u * N * d;
    float* op = opart + (long long)blockIdx.y * gridDim.x * N * d + base;
    for (int e = threadIdx.x; e < dd; e += TPB) W[e] = w0[(u % H) * dd + e];
    __syncthreads();
    const int nc = N / chunk;
    for (int ci = 0; ci < nc; ++ci) {
        const int c0 = (dir == 0 ? ci : nc - 1 - ci) * chunk;
        for (int e = threadIdx.x; e < dd; e += TPB) G[e] = 0.f;
        __syncthreads();
        for (int s0 = 0; s0 < chunk; s0 += CH_RB) {
            const int nr = min(CH_RB, chunk - s0);
            // residuals with W before this chunk's update
            for (int e = threadIdx.x; e < nr * d; e += TPB) {
                const int tt = e / d, j = e % d;
                const long long t = c0 + s0 + tt;
                float f = 0.f;
                for (int m = 0; m < d; ++m) f = fmaf(to_f(k[base + t * d + m]), W[m * d + j], f);
                R[e] = f - to_f(v[base + t * d + j]);
            }
            __syncthreads();
            for (int e = threadIdx.x; e < dd; e += TPB) {
                const int i = e / d, j = e % d;
                float g = G[e];
                for (int tt = 0; tt < nr; ++tt) g = fmaf(to_f(k[base + (long long)(c0 + s0 + tt) * d + i]), R[tt * d + j], g);
                G[e] = g;
            }
            __syncthreads();
        }
        for (int e = threadIdx.x; e < dd; e += TPB) W[e] -= eta_over_b * G[e];
        __syncthreads();
        // outputs of the chunk with the updated W
        for (int e = threadIdx.x; e < chunk * d; e += TPB) {
            const int tt = e / d, j = e % d;
            const long long t = c0 + tt;
            float s = 0.f;
            for (int m = 0; m < d; ++m) s = fmaf(to_f(q[base + t * d + m]), W[m * d + j], s);
            op[t * d + j] = s;
        }
        __syncthreads();
    }
}

template <typename T>
__global__ void __launch_bounds__(TPB) chunked_combine(const float* __restrict__ opart, T* __restrict__ out,
                                                       long long total, int nparts) {
    const long long e = (long long)blockIdx.x * TPB + threadIdx.x;
    if (e >= total) return;
    out[e] = from_f<T>(nparts == 2 ? opart[e] + opart[total + e] : opart[e]);
}

// ------------------------------------------------------------------ mini-batch training --
// One block per unit: E epochs over the chunks in raster order, W <- W - (eta/b) K_c^T (K_c W
// - V_c), nothing output per chunk; W_final (fp32) goes to wfin[u] (and w_out[u] if given).
template <typename T>
__global__ void __launch_bounds__(TPB) minibatch_train(const T* __restrict__ k, const T* __restrict__ v,
                                                       const float* __restrict__ w0, float* __restrict__ wfin,
                                                       float* __restrict__ w_out, int H, int N, int d, int chunk,
                                                       int epochs, float eta_over_b) {
    extern __shared__ float sm[];
    float* W = sm;
    float* G = W + d * d;
    float* R = G + d * d;
    const long long u = blockIdx.x;
    const int dd = d * d;
    const long long base = u * N * d;
    for (int e = threadIdx.x; e < dd; e += TPB) W[e] = w0[(u % H) * dd + e];
    __syncthreads();
    const int nc = N / chunk;
    for (int ep = 0; ep < epochs; ++ep)
        for (int ci = 0; ci < nc; ++ci) {
            const int c0 = ci * chunk;
            for (int e = threadIdx.x; e < dd; e += TPB) G[e] = 0.f;
            __syncthreads();
            for (int s0 = 0; s0 < chunk; s0 += CH_RB) {
                const int nr = min(CH_RB, chunk - s0);
                for (int e = threadIdx.x; e < nr * d; e += TPB) {  // residuals with W before the update
                    const int tt = e / d, j = e % d;
                    const long long t = c0 + s0 + tt;
                    float f = 0.f;
                    for (int m = 0; m < d; ++m) f = fmaf(to_f(k[base + t * d + m]), W[m * d + j], f);
                    R[e] = f - to_f(v[base + t * d + j]);
                }
                __syncthreads();
                for (int e = threadIdx.x; e < dd; e += TPB) {
                    const int i = e / d, j = e % d;
                    float g = G[e];
                    for (int tt = 0; tt < nr; ++tt) g = fmaf(to_f(k[base + (long long)(c0 + s0 + tt) * d + i]), R[tt * d + j], g);
                    G[e] = g;
                }
                __syncthreads();
            }
            for (int e = threadIdx.x; e < dd; e += TPB) W[e] -= eta_over_b * G[e];
            __syncthreads();
        }
    for (int e = threadIdx.x; e < dd; e += TPB) {
        wfin[u * dd + e] = W[e];
        if (w_out) w_out[u * dd + e] = W[e];
    }
}

// ------------------------------------------------------------------ TTT-Linear backward -
// Gradients of an outer loss through the full-batch step, for the upstream gradient dO:
//   M = Q^T dO,  W* = W0 - (eta/N)(G W0 - C),  A = W0 M^T + M W0^T (symmetric)
//   dQ = dO W*^T,  dV = (eta/N) K M,  dK = -(eta/N) (K A - V M^T),  dW0_u = M - (eta/N) G M
// (the chain rule back through o = q W*, W* = W0 - eta gW, gW = (1/N) sum k^T (k W0 - v)).
// gcm[u] = {G, C, M}, d x d each, token sums in fp64.
template <typename T>
__global__ void __launch_bounds__(TPB) linear_bwd_gram(const T* __restrict__ q, const T* __restrict__ k,
                                                       const T* __restrict__ v, const T* __restrict__ g,
                                                       float* __restrict__ gcm, int N, int d) {
    const long long u = blockIdx.x;
    const int e = blockIdx.y * TPB + threadIdx.x;
    const int dd = d * d;
    if (e >= 3 * dd) return;
    const int which = e / dd, r = (e % dd) / d, c = e % d;
    const T* a = (which == 2 ? q : k) + u * N * d;
    const T* b = (which == 0 ? k : which == 1 ? v : g) + u * N * d;
    double acc = 0.0;
    for (int t = 0; t < N; ++t)
        acc = fma((double)to_f(a[(long long)t * d + r]), (double)to_f(b[(long long)t * d + c]), acc);
    gcm[u * 3 * dd + e] = (float)acc;
}

// Per element (r, c) of unit u: wsa[u] = {W*, A}, dw0u[u] = dW0_u (fp32).
__global__ void __launch_bounds__(TPB) linear_bwd_finish(const float* __restrict__ gcm, const float* __restrict__ w0,
                                                         float* __restrict__ wsa, float* __restrict__ dw0u, int H,
                                                         int d, float eta_over_n) {
    const long long u = blockIdx.x;
    const int e = blockIdx.y * TPB + threadIdx.x;
    const int dd = d * d;
    if (e >= dd) return;
    const int r = e / d, c = e % d;
    const float* G = gcm + u * 3 * dd;
    const float* C = G + dd;
    const float* M = C + dd;
    const float* W0 = w0 + (u % H) * dd;
    float gw = 0.f, xrc = 0.f, xcr = 0.f, gm = 0.f;
    for (int m = 0; m < d; ++m) {
        gw = fmaf(G[r * d + m], W0[m * d + c], gw);
        xrc = fmaf(W0[r * d + m], M[c * d + m], xrc);
        xcr = fmaf(W0[c * d + m], M[r * d + m], xcr);
        gm = fmaf(G[r * d + m], M[m * d + c], gm);
    }
    wsa[u * 2 * dd + e] = W0[e] - eta_over_n * (gw - C[e]);
    wsa[u * 2 * dd + dd + e] = xrc + xcr;
    dw0u[u * dd + e] = M[e] - eta_over_n * gm;
}

// dQ, dK, dV at element (t, c)
template <typename T>
__global__ void __launch_bounds__(TPB) linear_bwd_apply(const T* __restrict__ k, const T* __restrict__ v,
                                                        const T* __restrict__ g, const float* __restrict__ gcm,
                                                        const float* __restrict__ wsa, T* __restrict__ dq,
                                                        T* __restrict__ dk, T* __restrict__ dv, int N, int d,
                                                        float eta_over_n) {
    const long long u = blockIdx.x;
    const long long e = (long long)blockIdx.y * TPB + threadIdx.x;
    if (e >= (long long)N * d) return;
    const long long t = e / d;
    const int c = (int)(e % d);
    const int dd = d * d;
    const float* M = gcm + u * 3 * dd + 2 * dd;
    const float* W = wsa + u * 2 * dd;
    const float* A = W + dd;
    const long long row = u * N * d + t * d;
    float sq = 0.f, sv = 0.f, ska = 0.f, skv = 0.f;
    for (int m = 0; m < d; ++m) {
        const float gm = to_f(g[row + m]), km = to_f(k[row + m]), vm = to_f(v[row + m]);
        sq = fmaf(gm, W[c * d + m], sq);   // dO W*^T
        sv = fmaf(km, M[m * d + c], sv);   // K M
        ska = fmaf(km, A[m * d + c], ska); // K A
        skv = fmaf(vm, M[c * d + m], skv); // V M^T
    }
    dq[row + c] = from_f<T>(sq);
    dv[row + c] = from_f<T>(eta_over_n * sv);
    dk[row + c] = from_f<T>(-eta_over_n * (ska - skv));
}

// dW0[h] = sum over batch entries b (in order) of dW0_(b, h)
__global__ void __launch_bounds__(TPB) linear_bwd_dw0(const float* __restrict__ dw0u, float* __restrict__ dw0, int B,
                                                      int H, int d) {
    const int h = blockIdx.x;
    const int e = blockIdx.y * blockDim.x + threadIdx.x;
    const int dd = d * d;
    griddep_wait();  // under programmatic dependent launch: the per-unit dW0 of the previous grid
    if (e >= dd) return;
    float s = 0.f;
    int b = 0;
    for (; b + 16 <= B; b += 16) {  // sixteen loads in flight, then the adds in batch order
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = dw0u[((long long)(b + i) * H + h) * dd + e];
#pragma unroll
        for (int i = 0; i < 16; ++i) s += x[i];
    }
    for (; b < B; ++b) s += dw0u[((long long)b * H + h) * dd + e];
    dw0[(long long)h * dd + e] = s;
}

// ------------------------------------------------------------------ ViT^3 block ---------
// [Q | K | V | G] = x Wqkvg at element (row R = b N + t, column j): Q, K, V head-split.
template <typename T>
__global__ void __launch_bounds__(TPB) block_proj(const T* __restrict__ x, const T* __restrict__ w, T* __restrict__ q,
                                                  T* __restrict__ k, T* __restrict__ v, T* __restrict__ g,
                                                  long long rows, int N, int C, int H) {
    const long long e = (long long)blockIdx.x * TPB + threadIdx.x;
    if (e >= rows * 4 * C) return;
    const long long R = e / (4 * C);
    const int j = (int)(e % (4 * C));
    float s = 0.f;
    for (int i = 0; i < C; ++i) s = fmaf(to_f(x[R * C + i]), to_f(w[(long long)i * 4 * C + j]), s);
    const int which = j / C, c = j % C, d = C / H;
    const long long b = R / N, t = R % N;
    if (which == 3) {
        g[R * C + c] = from_f<T>(s);
    } else {
        T* base = which == 0 ? q : which == 1 ? k : v;
        base[((b * H + c / d) * N + t) * d + c % d] = from_f<T>(s);
    }
}

// Z[R] = [O * sigmoid(G) | dwconv3x3(x)] (fp32) at element (R, j), j < 2C
template <typename T>
__global__ void __launch_bounds__(TPB) block_z(const T* __restrict__ x, const T* __restrict__ o,
                                               const T* __restrict__ g, const float* __restrict__ wc,
                                               float* __restrict__ z, long long rows, int N, int Hg, int Wg, int C,
                                               int H) {
    const long long e = (long long)blockIdx.x * TPB + threadIdx.x;
    if (e >= rows * 2 * C) return;
    const long long R = e / (2 * C);
    const int j = (int)(e % (2 * C));
    const long long b = R / N, t = R % N;
    const int d = C / H;
    if (j < C) {
        const float gv = to_f(g[R * C + j]);
        z[e] = to_f(o[((b * H + j / d) * N + t) * d + j % d]) / (1.f + expf(-gv));
    } else {
        const int c = j - C, py = (int)(t / Wg), px = (int)(t % Wg);
        float acc = 0.f;
        for (int a = 0; a < 3; ++a)
            for (int bb = 0; bb < 3; ++bb) {
                const int yy = py + a - 1, xx = px + bb - 1;
                if (yy >= 0 && yy < Hg && xx >= 0 && xx < Wg)
                    acc = fmaf(wc[c * 9 + a * 3 + bb], to_f(x[(b * N + (long long)yy * Wg + xx) * C + c]), acc);
            }
        z[e] = acc;
    }
}

// y = Z Wo at element (R, j)
template <typename T>
__global__ void __launch_bounds__(TPB) block_outproj(const float* __restrict__ z, const T* __restrict__ wo,
                                                     T* __restrict__ y, long long rows, int C) {
    const long long e = (long long)blockIdx.x * TPB + threadIdx.x;
    if (e >= rows * C) return;
    const long long R = e / C;
    const int j = (int)(e % C);
    float s = 0.f;
    for (int i = 0; i < 2 * C; ++i) s = fmaf(z[R * 2 * C + i], to_f(wo[(long long)i * C + j]), s);
    y[e] = from_f<T>(s);
}

// ------------------------------------------------------------------ conv preprocessing --
// x' = 3x3 depthwise conv of x over the Hg x Wg token grid of each unit (zero padding, no
// bias): one filter per feature of each head, taps w [H][d][3][3]; x, y [U][Hg*Wg][d].
template <typename T>
__global__ void __launch_bounds__(TPB) dwconv_prep(const T* __restrict__ x, const float* __restrict__ w,
                                                   T* __restrict__ y, int H, int Hg, int Wg, int d) {
    const long long u = blockIdx.x;
    const long long e = (long long)blockIdx.y * TPB + threadIdx.x;
    const long long N = (long long)Hg * Wg;
    if (e >= N * d) return;
    const int f = (int)(e % d);
    const long long t = e / d;
    const int py = (int)(t / Wg), px = (int)(t % Wg);
    const float* wf = w + ((u % H) * d + f) * 9;
    const T* xu = x + u * N * d;
    float acc = 0.f;
#pragma unroll
    for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int b = 0; b < 3; ++b) {
            const int yy = py + a - 1, xx = px + b - 1;
            if (yy >= 0 && yy < Hg && xx >= 0 && xx < Wg)
                acc = fmaf(wf[a * 3 + b], to_f(xu[((long long)yy * Wg + xx) * d + f]), acc);
        }
    y[u * N * d + e] = from_f<T>(acc);
}

// bf16 version for d % 8 == 0: one thread makes 8 consecutive features of one token (16-byte
// loads of the 3x3 neighbourhood, the head's filters staged in shared memory); blockIdx.z picks
// K (0) or V (1), so one launch preprocesses both.
__global__ void __launch_bounds__(TPB) dwconv_prep2_bf16(const __nv_bfloat16* __restrict__ k,
                                                         const __nv_bfloat16* __restrict__ v,
                                                         const float* __restrict__ wk, const float* __restrict__ wv,
                                                         __nv_bfloat16* __restrict__ kp, __nv_bfloat16* __restrict__ vp,
                                                         int H, int Hg, int Wg, int d) {
    extern __shared__ float wsm[];  // [d][9]
    const long long u = blockIdx.x;
    const bool isv = blockIdx.z != 0;
    const float* w = (isv ? wv : wk) + (u % H) * d * 9;
    for (int e = threadIdx.x; e < d * 9; e += TPB) wsm[e] = w[e];
    __syncthreads();
    const long long N = (long long)Hg * Wg;
    const int g8 = d / 8;
    const long long e = (long long)blockIdx.y * TPB + threadIdx.x;  // (token, 8-feature group)
    if (e >= N * g8) return;
    const long long t = e / g8;
    const int f0 = (int)(e % g8) * 8;
    const int py = (int)(t / Wg), px = (int)(t % Wg);
    const __nv_bfloat16* xu = (isv ? v : k) + u * N * d;
    float acc[8] = {};
#pragma unroll
    for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int b = 0; b < 3; ++b) {
            const int yy = py + a - 1, xx = px + b - 1;
            if (yy < 0 || yy >= Hg || xx < 0 || xx >= Wg) continue;
            const uint4 raw = *reinterpret_cast<const uint4*>(xu + ((long long)yy * Wg + xx) * d + f0);
            const __nv_bfloat162* pr = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(pr[i]);
                acc[2 * i] = fmaf(wsm[(f0 + 2 * i) * 9 + a * 3 + b], f.x, acc[2 * i]);
                acc[2 * i + 1] = fmaf(wsm[(f0 + 2 * i + 1) * 9 + a * 3 + b], f.y, acc[2 * i + 1]);
            }
        }
    *reinterpret_cast<uint4*>((isv ? vp : kp) + u * N * d + t * d + f0) =
        make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]), pack_bf16(acc[4], acc[5]),
                   pack_bf16(acc[6], acc[7]));
}

// bf16, d = 64: block (column chunk, row strip) of unit blockIdx.y; thread (column, feature
// group g) walks the strip's PS_ROWS rows with its 8 features' 72 filter taps in registers and
// their 3 x 3 neighbourhood in a window that slides down one row per output token (three
// 16-byte loads per output instead of nine).  A warp covers 4 consecutive tokens x 64 features:
// 512 contiguous bytes per load and per store.  blockIdx.z picks K (0) or V (1).  The sums run
// in the same order as dwconv_prep2_bf16 (tap row, tap column) with packed fp32 FMAs on feature
// pairs (fma.rn.f32x2: an IEEE fma per lane), so both give the same values.
constexpr int PS_ROWS = 8;
__global__ void __launch_bounds__(256, 2) dwconv_prep_strip_bf16(const __nv_bfloat16* __restrict__ k,
                                                              const __nv_bfloat16* __restrict__ v,
                                                              const float* __restrict__ wk, const float* __restrict__ wv,
                                                              __nv_bfloat16* __restrict__ kp,
                                                              __nv_bfloat16* __restrict__ vp, int H, int Hg, int Wg) {
    constexpr int D = 64;
    const int g = threadIdx.x & 7, c = threadIdx.x >> 3;
    const int nxc = (Wg + 31) / 32;
    const int x = (int)(blockIdx.x % nxc) * 32 + c;
    const int y0 = (int)(blockIdx.x / nxc) * PS_ROWS;
    if (x >= Wg) return;  // no barrier below
    const long long u = blockIdx.y;
    const bool isv = blockIdx.z != 0;
    const long long N = (long long)Hg * Wg;
    const float* w = (isv ? wv : wk) + ((u % H) * D + g * 8) * 9;  // [8 features][9 taps]
    uint64_t wr[4][9];  // taps of features (2i, 2i + 1) as packed fp32 pairs
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int t = 0; t < 9; ++t)
            wr[i][t] = (uint64_t)__float_as_uint(__ldg(w + 2 * i * 9 + t)) |
                       ((uint64_t)__float_as_uint(__ldg(w + (2 * i + 1) * 9 + t)) << 32);
    const __nv_bfloat16* xu = (isv ? v : k) + u * N * D + g * 8;
    __nv_bfloat16* ou = (isv ? vp : kp) + u * N * D + g * 8;
    auto ld = [&](int yy, int xx) -> uint4 {
        return (yy >= 0 && yy < Hg && xx >= 0 && xx < Wg)
                   ? *reinterpret_cast<const uint4*>(xu + ((long long)yy * Wg + xx) * D)
                   : make_uint4(0, 0, 0, 0);
    };
    uint4 win[3][3];  // rows y - 1, y, y + 1; columns x - 1, x, x + 1
#pragma unroll
    for (int b = 0; b < 3; ++b) {
        win[0][b] = ld(y0 - 1, x + b - 1);
        win[1][b] = ld(y0, x + b - 1);
        win[2][b] = ld(y0 + 1, x + b - 1);
    }
    const int y1 = min(y0 + PS_ROWS, Hg);
    for (int y = y0; y < y1; ++y) {
        uint4 nxt[3];  // row y + 2, requested before this row's arithmetic
#pragma unroll
        for (int b = 0; b < 3; ++b) nxt[b] = y + 1 < y1 ? ld(y + 2, x + b - 1) : make_uint4(0, 0, 0, 0);
        uint64_t acc[4] = {0, 0, 0, 0};  // features (2i, 2i + 1), packed fp32
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int b = 0; b < 3; ++b) {
                const uint32_t wv4[4] = {win[a][b].x, win[a][b].y, win[a][b].z, win[a][b].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    // bf16 pair -> fp32 pair: low half to the high 16 bits of the first word
                    const uint64_t f = (uint64_t)(wv4[i] << 16) | ((uint64_t)(wv4[i] & 0xffff0000u) << 32);
                    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc[i]) : "l"(wr[i][a * 3 + b]), "l"(f));
                }
            }
        *reinterpret_cast<uint4*>(ou + ((long long)y * Wg + x) * D) =
            make_uint4(pack_bf16(__uint_as_float((uint32_t)acc[0]), __uint_as_float((uint32_t)(acc[0] >> 32))),
                       pack_bf16(__uint_as_float((uint32_t)acc[1]), __uint_as_float((uint32_t)(acc[1] >> 32))),
                       pack_bf16(__uint_as_float((uint32_t)acc[2]), __uint_as_float((uint32_t)(acc[2] >> 32))),
                       pack_bf16(__uint_as_float((uint32_t)acc[3]), __uint_as_float((uint32_t)(acc[3] >> 32))));
#pragma unroll
        for (int b = 0; b < 3; ++b) {
            win[0][b] = win[1][b];
            win[1][b] = win[2][b];
            win[2][b] = nxt[b];
        }
    }
}

}  // namespace simt
