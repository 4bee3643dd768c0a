/*
 * ttt_oracle.c -- plain, slow, fp64 CPU oracle for the Test-Time-Training (TTT) layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this
 * file: only the test-suite, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header or constant table with the CUDA library.
 *
 * What it computes (per (batch, head) unit, or per (image, channel) for the conv model):
 *   the layer of "ViT^3: Unlocking Test-Time Training in Vision" (techloop.online blog,
 *   section "核心想法：把 attention 改写成 online learning", steps 1-3): train an inner
 *   model F_W on the pairs (k_i, v_i), obtain W*, output F_{W*}(q_i).
 *   Inner training follows the same blog's design-study summary ("inner training 怎么配"):
 *   a single epoch over the full batch with inner learning rate 1.0, and no L1-type loss.
 *   The loss is l(W) = (1/N) * sum_i 1/2 * ||F_W(k_i) - v_i||^2 and the step is
 *   W* = W0 - eta * grad l(W0).  The gradient is derived by hand (the blog's note that the
 *   official code writes the closed-form gradient instead of calling autograd).
 *
 * Inner models:
 *   - linear:      F_W(x) = x W                       (TTT-Linear, Sun et al. abstract)
 *   - two-layer MLP: F(x) = gelu_tanh(x W1) W2, no biases (TTT-MLP, Sun et al. abstract)
 *   - 3x3 depthwise conv on the token grid, zero padding, no bias (ViT^3 blog, the
 *     "3x3 depthwise conv" inner module of the design-study section)
 *   - chunked online variant: W_t = W_{t-1} - eta * grad l(W_{t-1}; x_t) applied per chunk of b
 *     tokens (Vision-TTT gist, "Technische samenvatting", item 1 and item 3: mini-batches),
 *     scanned in raster and reverse-raster order (same page, item 2: bidirectional scan),
 *     the two outputs summed.
 *
 * Readings where the pages are silent (each is listed with its reason in the design notes):
 *   loss normalised by 1/N; W0 shared per head across the batch; cross-correlation with tap
 *   (a,b) <-> offset (a-1, b-1); chunk step normalised by 1/b; the chunk output uses W after
 *   that chunk's update; both scan directions start from W0.
 *
 * Everything is computed in double with explicit per-token loops and no BLAS.
 * All arrays are dense row-major; see the prototypes in ttt_oracle.h.
 * Parity status: every function here is pinned by the CPU test-suite (closed forms,
 * finite differences, autograd of library operators, special cases, hand-worked examples).
 */
#include "ttt_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------ */
/* Thread pool over independent units: each unit is computed by exactly one thread.      */
/* ------------------------------------------------------------------------------------ */
typedef void (*unit_fn)(const void* ctx, long unit);

typedef struct {
    const void* ctx;
    unit_fn fn;
    long n_units;
    long next;
    pthread_mutex_t lock;
} pool_t;

static void* pool_worker(void* arg) {
    pool_t* p = (pool_t*)arg;
    for (;;) {
        long u;
        pthread_mutex_lock(&p->lock);
        u = p->next++;
        pthread_mutex_unlock(&p->lock);
        if (u >= p->n_units) break;
        p->fn(p->ctx, u);
    }
    return NULL;
}

static void run_units(long n_units, int threads, unit_fn fn, const void* ctx) {
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    if ((long)threads > n_units) threads = (int)(n_units > 0 ? n_units : 1);
    pool_t p;
    p.ctx = ctx;
    p.fn = fn;
    p.n_units = n_units;
    p.next = 0;
    pthread_mutex_init(&p.lock, NULL);
    if (threads == 1) {
        pool_worker(&p);
    } else {
        pthread_t tid[256];
        for (int t = 0; t < threads; ++t) pthread_create(&tid[t], NULL, pool_worker, &p);
        for (int t = 0; t < threads; ++t) pthread_join(tid[t], NULL);
    }
    pthread_mutex_destroy(&p.lock);
}

/* ==================================================================================== */
/* TTT-Linear: F_W(x) = x W, W is d x d.                                                */
/* ==================================================================================== */

double ttt_oracle_linear_loss(const double* k, const double* v, const double* w, int N, int d) {
    double total = 0.0;
    for (int t = 0; t < N; ++t) {
        for (int j = 0; j < d; ++j) {
            double f = 0.0;
            for (int m = 0; m < d; ++m) f += k[(long)t * d + m] * w[(long)m * d + j];
            double r = f - v[(long)t * d + j];
            total += 0.5 * r * r;
        }
    }
    return total / (double)N;
}

void ttt_oracle_linear_grad(const double* k, const double* v, const double* w, int N, int d,
                            double* g) {
    double* r = (double*)malloc(sizeof(double) * (size_t)d);
    memset(g, 0, sizeof(double) * (size_t)d * d);
    for (int t = 0; t < N; ++t) {
        const double* kt = k + (long)t * d;
        const double* vt = v + (long)t * d;
        /* residual of token t: r = k_t W - v_t */
        for (int j = 0; j < d; ++j) {
            double f = 0.0;
            for (int m = 0; m < d; ++m) f += kt[m] * w[(long)m * d + j];
            r[j] = f - vt[j];
        }
        /* d/dW of 1/2 ||k_t W - v_t||^2 is the outer product k_t^T r */
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) g[(long)i * d + j] += kt[i] * r[j];
    }
    for (long e = 0; e < (long)d * d; ++e) g[e] /= (double)N;
    free(r);
}

/* o_t = x_t W for every token of one unit */
static void linear_apply(const double* x, const double* w, int N, int d, double* o) {
    for (int t = 0; t < N; ++t)
        for (int j = 0; j < d; ++j) {
            double s = 0.0;
            for (int m = 0; m < d; ++m) s += x[(long)t * d + m] * w[(long)m * d + j];
            o[(long)t * d + j] = s;
        }
}

typedef struct {
    const double *q, *k, *v, *w0;
    double *out, *w_star;
    int H, N, d;
    double eta;
} linear_ctx;

static void linear_unit(const void* vctx, long u) {
    const linear_ctx* c = (const linear_ctx*)vctx;
    const int d = c->d, N = c->N;
    const long h = u % c->H;
    const long tok = (long)N * d;
    const double* w0 = c->w0 + h * (long)d * d;
    double* g = (double*)malloc(sizeof(double) * (size_t)d * d);
    double* ws = (double*)malloc(sizeof(double) * (size_t)d * d);
    ttt_oracle_linear_grad(c->k + u * tok, c->v + u * tok, w0, N, d, g);
    for (long e = 0; e < (long)d * d; ++e) ws[e] = w0[e] - c->eta * g[e];
    linear_apply(c->q + u * tok, ws, N, d, c->out + u * tok);
    if (c->w_star) memcpy(c->w_star + u * (long)d * d, ws, sizeof(double) * (size_t)d * d);
    free(g);
    free(ws);
}

int ttt_oracle_linear_fullbatch(const double* q, const double* k, const double* v,
                                const double* w0, double* out, double* w_star, int B, int H,
                                int N, int d, double eta, int threads) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 1;
    linear_ctx c = {q, k, v, w0, out, w_star, H, N, d, eta};
    run_units((long)B * H, threads, linear_unit, &c);
    return 0;
}

/* ==================================================================================== */
/* 3x3 depthwise-conv inner model on an Hg x Wg token grid, channels-last [Hg, Wg, C].   */
/* F_w(K)_c(y, x) = sum_{a,b in 0..2} w[c][a][b] * K_c(y + a - 1, x + b - 1), zero pad. */
/* ==================================================================================== */

static double grid_at(const double* x, int Hg, int Wg, int C, int y, int xx, int c) {
    if (y < 0 || y >= Hg || xx < 0 || xx >= Wg) return 0.0;
    return x[((long)y * Wg + xx) * C + c];
}

/* forward of the conv model for one image and one channel at one pixel */
static double dwconv_at(const double* x, const double* wc, int Hg, int Wg, int C, int y,
                        int xx, int c) {
    double s = 0.0;
    for (int a = 0; a < 3; ++a)
        for (int b = 0; b < 3; ++b)
            s += wc[a * 3 + b] * grid_at(x, Hg, Wg, C, y + a - 1, xx + b - 1, c);
    return s;
}

double ttt_oracle_dwconv_loss(const double* k, const double* v, const double* w, int Hg,
                              int Wg, int C) {
    const long N = (long)Hg * Wg;
    double total = 0.0;
    for (int y = 0; y < Hg; ++y)
        for (int x = 0; x < Wg; ++x)
            for (int c = 0; c < C; ++c) {
                double r = dwconv_at(k, w + c * 9, Hg, Wg, C, y, x, c) -
                           v[((long)y * Wg + x) * C + c];
                total += 0.5 * r * r;
            }
    return total / (double)N;
}

/* gradient for one channel c of one image: g[9] */
static void dwconv_grad_channel(const double* k, const double* v, const double* wc, int Hg,
                                int Wg, int C, int c, double* g) {
    const long N = (long)Hg * Wg;
    for (int e = 0; e < 9; ++e) g[e] = 0.0;
    for (int y = 0; y < Hg; ++y)
        for (int x = 0; x < Wg; ++x) {
            double r = dwconv_at(k, wc, Hg, Wg, C, y, x, c) - v[((long)y * Wg + x) * C + c];
            for (int a = 0; a < 3; ++a)
                for (int b = 0; b < 3; ++b)
                    g[a * 3 + b] += r * grid_at(k, Hg, Wg, C, y + a - 1, x + b - 1, c);
        }
    for (int e = 0; e < 9; ++e) g[e] /= (double)N;
}

void ttt_oracle_dwconv_grad(const double* k, const double* v, const double* w, int Hg, int Wg,
                            int C, double* g) {
    for (int c = 0; c < C; ++c) dwconv_grad_channel(k, v, w + c * 9, Hg, Wg, C, c, g + c * 9);
}

typedef struct {
    const double *q, *k, *v, *w0;
    double *out, *w_star;
    int Hg, Wg, C;
    double eta;
} dwconv_ctx;

static void dwconv_unit(const void* vctx, long u) {
    const dwconv_ctx* c = (const dwconv_ctx*)vctx;
    const int C = c->C, Hg = c->Hg, Wg = c->Wg;
    const long b = u / C;
    const int ch = (int)(u % C);
    const long img = (long)Hg * Wg * C;
    const double* k = c->k + b * img;
    const double* v = c->v + b * img;
    const double* q = c->q + b * img;
    double g[9], ws[9];
    dwconv_grad_channel(k, v, c->w0 + ch * 9, Hg, Wg, C, ch, g);
    for (int e = 0; e < 9; ++e) ws[e] = c->w0[ch * 9 + e] - c->eta * g[e];
    for (int y = 0; y < Hg; ++y)
        for (int x = 0; x < Wg; ++x)
            c->out[b * img + ((long)y * Wg + x) * C + ch] = dwconv_at(q, ws, Hg, Wg, C, y, x, ch);
    if (c->w_star)
        for (int e = 0; e < 9; ++e) c->w_star[(b * C + ch) * 9 + e] = ws[e];
}

int ttt_oracle_dwconv_fullbatch(const double* q, const double* k, const double* v,
                                const double* w0, double* out, double* w_star, int B, int Hg,
                                int Wg, int C, double eta, int threads) {
    if (B <= 0 || Hg <= 0 || Wg <= 0 || C <= 0) return 1;
    dwconv_ctx c = {q, k, v, w0, out, w_star, Hg, Wg, C, eta};
    run_units((long)B * C, threads, dwconv_unit, &c);
    return 0;
}

/* ==================================================================================== */
/* TTT-MLP: F(x) = gelu_tanh(x W1) W2, W1 is d x h, W2 is h x d, no biases.             */
/* gelu_tanh(u) = u/2 * (1 + tanh(sqrt(2/pi) * (u + 0.044715 u^3)))  (Hendrycks & Gimpel)*/
/* ==================================================================================== */

static const double kGeluA = 0.044715;

static double gelu_s(void) { return sqrt(2.0 / 3.14159265358979323846); }

double ttt_oracle_gelu_tanh(double u) {
    double t = tanh(gelu_s() * (u + kGeluA * u * u * u));
    return 0.5 * u * (1.0 + t);
}

/* derivative by the product and chain rules, using the same t */
double ttt_oracle_gelu_tanh_grad(double u) {
    double s = gelu_s();
    double t = tanh(s * (u + kGeluA * u * u * u));
    return 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * s * (1.0 + 3.0 * kGeluA * u * u);
}

double ttt_oracle_mlp_loss(const double* k, const double* v, const double* w1,
                           const double* w2, int N, int d, int h) {
    double* a = (double*)malloc(sizeof(double) * (size_t)h);
    double total = 0.0;
    for (int t = 0; t < N; ++t) {
        const double* kt = k + (long)t * d;
        for (int m = 0; m < h; ++m) {
            double z = 0.0;
            for (int i = 0; i < d; ++i) z += kt[i] * w1[(long)i * h + m];
            a[m] = ttt_oracle_gelu_tanh(z);
        }
        for (int j = 0; j < d; ++j) {
            double p = 0.0;
            for (int m = 0; m < h; ++m) p += a[m] * w2[(long)m * d + j];
            double r = p - v[(long)t * d + j];
            total += 0.5 * r * r;
        }
    }
    free(a);
    return total / (double)N;
}

void ttt_oracle_mlp_grad(const double* k, const double* v, const double* w1, const double* w2,
                         int N, int d, int h, double* g1, double* g2) {
    double* z = (double*)malloc(sizeof(double) * (size_t)h);
    double* a = (double*)malloc(sizeof(double) * (size_t)h);
    double* r = (double*)malloc(sizeof(double) * (size_t)d);
    memset(g1, 0, sizeof(double) * (size_t)d * h);
    memset(g2, 0, sizeof(double) * (size_t)h * d);
    for (int t = 0; t < N; ++t) {
        const double* kt = k + (long)t * d;
        /* forward: z = k_t W1, a = gelu(z), p = a W2, r = p - v_t */
        for (int m = 0; m < h; ++m) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += kt[i] * w1[(long)i * h + m];
            z[m] = s;
            a[m] = ttt_oracle_gelu_tanh(s);
        }
        for (int j = 0; j < d; ++j) {
            double p = 0.0;
            for (int m = 0; m < h; ++m) p += a[m] * w2[(long)m * d + j];
            r[j] = p - v[(long)t * d + j];
        }
        /* backward of 1/2 ||r||^2: dW2 = a^T r, da = r W2^T, dz = da * gelu'(z), dW1 = k^T dz */
        for (int m = 0; m < h; ++m) {
            double da = 0.0;
            for (int j = 0; j < d; ++j) {
                g2[(long)m * d + j] += a[m] * r[j];
                da += r[j] * w2[(long)m * d + j];
            }
            double dz = da * ttt_oracle_gelu_tanh_grad(z[m]);
            for (int i = 0; i < d; ++i) g1[(long)i * h + m] += kt[i] * dz;
        }
    }
    for (long e = 0; e < (long)d * h; ++e) {
        g1[e] /= (double)N;
        g2[e] /= (double)N;
    }
    free(z);
    free(a);
    free(r);
}

typedef struct {
    const double *q, *k, *v, *w1, *w2;
    double *out, *w1_star, *w2_star;
    int H, N, d, h;
    double eta;
} mlp_ctx;

static void mlp_unit(const void* vctx, long u) {
    const mlp_ctx* c = (const mlp_ctx*)vctx;
    const int d = c->d, h = c->h, N = c->N;
    const long hd = u % c->H;
    const long tok = (long)N * d;
    const long wsz = (long)d * h;
    const double* w1 = c->w1 + hd * wsz;
    const double* w2 = c->w2 + hd * wsz;
    double* g1 = (double*)malloc(sizeof(double) * (size_t)wsz);
    double* g2 = (double*)malloc(sizeof(double) * (size_t)wsz);
    double* w1s = (double*)malloc(sizeof(double) * (size_t)wsz);
    double* w2s = (double*)malloc(sizeof(double) * (size_t)wsz);
    double* a = (double*)malloc(sizeof(double) * (size_t)h);
    ttt_oracle_mlp_grad(c->k + u * tok, c->v + u * tok, w1, w2, N, d, h, g1, g2);
    for (long e = 0; e < wsz; ++e) {
        w1s[e] = w1[e] - c->eta * g1[e];
        w2s[e] = w2[e] - c->eta * g2[e];
    }
    const double* q = c->q + u * tok;
    double* o = c->out + u * tok;
    for (int t = 0; t < N; ++t) {
        for (int m = 0; m < h; ++m) {
            double z = 0.0;
            for (int i = 0; i < d; ++i) z += q[(long)t * d + i] * w1s[(long)i * h + m];
            a[m] = ttt_oracle_gelu_tanh(z);
        }
        for (int j = 0; j < d; ++j) {
            double s = 0.0;
            for (int m = 0; m < h; ++m) s += a[m] * w2s[(long)m * d + j];
            o[(long)t * d + j] = s;
        }
    }
    if (c->w1_star) memcpy(c->w1_star + u * wsz, w1s, sizeof(double) * (size_t)wsz);
    if (c->w2_star) memcpy(c->w2_star + u * wsz, w2s, sizeof(double) * (size_t)wsz);
    free(g1);
    free(g2);
    free(w1s);
    free(w2s);
    free(a);
}

int ttt_oracle_mlp_fullbatch(const double* q, const double* k, const double* v,
                             const double* w1, const double* w2, double* out, double* w1_star,
                             double* w2_star, int B, int H, int N, int d, int h, double eta,
                             int threads) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || h <= 0) return 1;
    mlp_ctx c = {q, k, v, w1, w2, out, w1_star, w2_star, H, N, d, h, eta};
    run_units((long)B * H, threads, mlp_unit, &c);
    return 0;
}

/* ==================================================================================== */
/* Chunked online TTT-Linear, scanned forward and backward.                             */
/* One direction over a token sequence x_0..x_{N-1} (chunks of b consecutive tokens):    */
/*   W <- W0; for each chunk c in order:                                                 */
/*       G_c = sum_{t in c} k_t^T (k_t W - v_t)      (residuals with W before the update) */
/*       W  <- W - (eta / b) G_c                                                          */
/*       o_t = q_t W for t in c                        (W after the chunk's update)       */
/* The reverse direction is the same scan run on the reversed sequence, its outputs put  */
/* back in the original order.  direction: +1 forward, -1 reverse, 0 both summed.       */
/* ==================================================================================== */

/* forward scan of one sequence given by an index map idx[t] (token t of the scan is row idx[t]) */
static void chunked_scan(const double* q, const double* k, const double* v, const double* w0,
                         const int* idx, int N, int d, int b, double eta, double* o_acc) {
    double* w = (double*)malloc(sizeof(double) * (size_t)d * d);
    double* gc = (double*)malloc(sizeof(double) * (size_t)d * d);
    double* r = (double*)malloc(sizeof(double) * (size_t)d);
    memcpy(w, w0, sizeof(double) * (size_t)d * d);
    for (int c0 = 0; c0 < N; c0 += b) {
        int c1 = c0 + b < N ? c0 + b : N;
        memset(gc, 0, sizeof(double) * (size_t)d * d);
        for (int s = c0; s < c1; ++s) {
            const double* kt = k + (long)idx[s] * d;
            const double* vt = v + (long)idx[s] * d;
            for (int j = 0; j < d; ++j) {
                double f = 0.0;
                for (int m = 0; m < d; ++m) f += kt[m] * w[(long)m * d + j];
                r[j] = f - vt[j];
            }
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j) gc[(long)i * d + j] += kt[i] * r[j];
        }
        for (long e = 0; e < (long)d * d; ++e) w[e] -= (eta / (double)b) * gc[e];
        for (int s = c0; s < c1; ++s) {
            const double* qt = q + (long)idx[s] * d;
            double* ot = o_acc + (long)idx[s] * d;
            for (int j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int m = 0; m < d; ++m) acc += qt[m] * w[(long)m * d + j];
                ot[j] += acc;
            }
        }
    }
    free(w);
    free(gc);
    free(r);
}

typedef struct {
    const double *q, *k, *v, *w0;
    double* out;
    int H, N, d, b, direction;
    double eta;
} chunked_ctx;

static void chunked_unit(const void* vctx, long u) {
    const chunked_ctx* c = (const chunked_ctx*)vctx;
    const int d = c->d, N = c->N;
    const long h = u % c->H;
    const long tok = (long)N * d;
    const double* w0 = c->w0 + h * (long)d * d;
    int* idx = (int*)calloc((size_t)N, sizeof(int));
    double* o = c->out + u * tok;
    memset(o, 0, sizeof(double) * (size_t)tok);
    if (c->direction >= 0) {
        for (int t = 0; t < N; ++t) idx[t] = t; /* raster order */
        chunked_scan(c->q + u * tok, c->k + u * tok, c->v + u * tok, w0, idx, N, d, c->b,
                     c->eta, o);
    }
    if (c->direction <= 0) {
        for (int t = 0; t < N; ++t) idx[t] = N - 1 - t; /* reverse raster order */
        chunked_scan(c->q + u * tok, c->k + u * tok, c->v + u * tok, w0, idx, N, d, c->b,
                     c->eta, o);
    }
    free(idx);
}

int ttt_oracle_linear_chunked(const double* q, const double* k, const double* v,
                              const double* w0, double* out, int B, int H, int N, int d,
                              int chunk, double eta, int direction, int threads) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || chunk <= 0) return 1;
    if (direction < -1 || direction > 1) return 1;
    chunked_ctx c = {q, k, v, w0, out, H, N, d, chunk, direction, eta};
    run_units((long)B * H, threads, chunked_unit, &c);
    return 0;
}

/* ==================================================================================== */
/* Backward of TTT-Linear full batch (outer training through the inner step).          */
/* Forward, per unit:  r_i = k_i W0 - v_i,  gW = (1/N) sum_i k_i^T r_i,                  */
/*                     W* = W0 - eta gW,   o_j = q_j W*.                                 */
/* Given the upstream gradient g_j = dL/do_j, the chain rule taken step by step back     */
/* through those four lines (written out by hand, as the ViT^3 blog notes the official   */
/* code does for the inner step, "从官方代码看…", third point):                            */
/*   dW*    = sum_j q_j^T g_j            dq_j = g_j W*^T                                 */
/*   dgW    = -eta dW*                   dW0 += dW*            (W* = W0 - eta gW)        */
/*   dr_i   = (1/N) k_i dgW              dk_i += (1/N) r_i dgW^T   (gW = mean k^T r)     */
/*   dk_i  += dr_i W0^T                  dv_i  = -dr_i          dW0 += k_i^T dr_i        */
/* W0 is shared by the batch entries of a head, so dW0[h] = sum over b (b ascending).    */
/* ==================================================================================== */

typedef struct {
    const double *q, *k, *v, *w0, *dout;
    double *dq, *dk, *dv, *dw0_unit;
    int H, N, d;
    double eta;
} linear_bwd_ctx;

static void linear_bwd_unit(const void* vctx, long u) {
    const linear_bwd_ctx* c = (const linear_bwd_ctx*)vctx;
    const int d = c->d, N = c->N;
    const long h = u % c->H;
    const long tok = (long)N * d;
    const long dd = (long)d * d;
    const double* w0 = c->w0 + h * dd;
    const double *q = c->q + u * tok, *k = c->k + u * tok, *v = c->v + u * tok;
    const double* g = c->dout + u * tok;
    double *dq = c->dq + u * tok, *dk = c->dk + u * tok, *dv = c->dv + u * tok;
    double* dw0 = c->dw0_unit + u * dd;
    double* gw = (double*)malloc(sizeof(double) * (size_t)dd);
    double* ws = (double*)malloc(sizeof(double) * (size_t)dd);
    double* dws = (double*)calloc((size_t)dd, sizeof(double));
    double* dgw = (double*)malloc(sizeof(double) * (size_t)dd);
    double* r = (double*)malloc(sizeof(double) * (size_t)d);
    double* dr = (double*)malloc(sizeof(double) * (size_t)d);
    /* forward: gW and W* */
    ttt_oracle_linear_grad(k, v, w0, N, d, gw);
    for (long e = 0; e < dd; ++e) ws[e] = w0[e] - c->eta * gw[e];
    /* o_j = q_j W*:  dW* = sum_j q_j^T g_j,  dq_j = g_j W*^T */
    for (int t = 0; t < N; ++t) {
        const double* qt = q + (long)t * d;
        const double* gt = g + (long)t * d;
        for (int a = 0; a < d; ++a)
            for (int b = 0; b < d; ++b) dws[(long)a * d + b] += qt[a] * gt[b];
        for (int a = 0; a < d; ++a) {
            double s = 0.0;
            for (int b = 0; b < d; ++b) s += gt[b] * ws[(long)a * d + b];
            dq[(long)t * d + a] = s;
        }
    }
    /* W* = W0 - eta gW */
    for (long e = 0; e < dd; ++e) {
        dgw[e] = -c->eta * dws[e];
        dw0[e] = dws[e];
    }
    /* gW = (1/N) sum_i k_i^T r_i with r_i = k_i W0 - v_i, token by token */
    for (int t = 0; t < N; ++t) {
        const double* kt = k + (long)t * d;
        const double* vt = v + (long)t * d;
        for (int j = 0; j < d; ++j) {
            double f = 0.0;
            for (int m = 0; m < d; ++m) f += kt[m] * w0[(long)m * d + j];
            r[j] = f - vt[j];
        }
        for (int b = 0; b < d; ++b) { /* dr_i = (1/N) k_i dgW */
            double s = 0.0;
            for (int a = 0; a < d; ++a) s += kt[a] * dgw[(long)a * d + b];
            dr[b] = s / (double)N;
        }
        for (int a = 0; a < d; ++a) {
            double s1 = 0.0, s2 = 0.0;
            for (int b = 0; b < d; ++b) {
                s1 += dgw[(long)a * d + b] * r[b];   /* (1/N) (r_i dgW^T)_a */
                s2 += dr[b] * w0[(long)a * d + b];   /* (dr_i W0^T)_a      */
            }
            dk[(long)t * d + a] = s1 / (double)N + s2;
        }
        for (int b = 0; b < d; ++b) dv[(long)t * d + b] = -dr[b];
        for (int a = 0; a < d; ++a)
            for (int b = 0; b < d; ++b) dw0[(long)a * d + b] += kt[a] * dr[b];
    }
    free(gw);
    free(ws);
    free(dws);
    free(dgw);
    free(r);
    free(dr);
}

int ttt_oracle_linear_fullbatch_bwd(const double* q, const double* k, const double* v,
                                    const double* w0, const double* dout, double* dq,
                                    double* dk, double* dv, double* dw0, int B, int H, int N,
                                    int d, double eta, int threads) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 1;
    const long dd = (long)d * d;
    double* per_unit = (double*)malloc(sizeof(double) * (size_t)B * H * dd);
    if (!per_unit) return 1;
    linear_bwd_ctx c = {q, k, v, w0, dout, dq, dk, dv, per_unit, H, N, d, eta};
    run_units((long)B * H, threads, linear_bwd_unit, &c);
    for (int h = 0; h < H; ++h)
        for (long e = 0; e < dd; ++e) {
            double s = 0.0;
            for (int b = 0; b < B; ++b) s += per_unit[((long)b * H + h) * dd + e];
            dw0[h * dd + e] = s;
        }
    free(per_unit);
    return 0;
}

/* ==================================================================================== */
/* Mini-batch / multi-epoch inner training, then the trained model applied to Q.        */
/* The inner-training options the ViT^3 blog's design study varies ("inner training 怎么 */
/* 配": full batch or mini-batch, how many epochs): E epochs over the tokens in raster     */
/* order, each epoch a sequence of mini-batches of b consecutive tokens,                 */
/*     W <- W - (eta / b) sum_{t in chunk} k_t^T (k_t W - v_t)                            */
/* (the online update rule of the Vision-TTT gist, item 1, per mini-batch as in item 3), */
/* then o_t = q_t W_final for every token.  b = N and E = 1 is the full-batch step.      */
/* ==================================================================================== */

typedef struct {
    const double *q, *k, *v, *w0;
    double *out, *w_final;
    int H, N, d, b, epochs;
    double eta;
} minibatch_ctx;

static void minibatch_unit(const void* vctx, long u) {
    const minibatch_ctx* c = (const minibatch_ctx*)vctx;
    const int d = c->d, N = c->N, b = c->b;
    const long h = u % c->H;
    const long tok = (long)N * d;
    const long dd = (long)d * d;
    const double *k = c->k + u * tok, *v = c->v + u * tok;
    double* w = (double*)malloc(sizeof(double) * (size_t)dd);
    double* gc = (double*)malloc(sizeof(double) * (size_t)dd);
    double* r = (double*)malloc(sizeof(double) * (size_t)d);
    memcpy(w, c->w0 + h * dd, sizeof(double) * (size_t)dd);
    for (int e = 0; e < c->epochs; ++e)
        for (int c0 = 0; c0 < N; c0 += b) {
            memset(gc, 0, sizeof(double) * (size_t)dd);
            for (int t = c0; t < c0 + b; ++t) {
                const double* kt = k + (long)t * d;
                const double* vt = v + (long)t * d;
                for (int j = 0; j < d; ++j) {
                    double f = 0.0;
                    for (int m = 0; m < d; ++m) f += kt[m] * w[(long)m * d + j];
                    r[j] = f - vt[j];
                }
                for (int i = 0; i < d; ++i)
                    for (int j = 0; j < d; ++j) gc[(long)i * d + j] += kt[i] * r[j];
            }
            for (long x = 0; x < dd; ++x) w[x] -= (c->eta / (double)b) * gc[x];
        }
    linear_apply(c->q + u * tok, w, N, d, c->out + u * tok);
    if (c->w_final) memcpy(c->w_final + u * dd, w, sizeof(double) * (size_t)dd);
    free(w);
    free(gc);
    free(r);
}

int ttt_oracle_linear_minibatch(const double* q, const double* k, const double* v,
                                const double* w0, double* out, double* w_final, int B, int H,
                                int N, int d, int chunk, int epochs, double eta, int threads) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || chunk <= 0 || epochs <= 0) return 1;
    if (N % chunk != 0) return 1;
    minibatch_ctx c = {q, k, v, w0, out, w_final, H, N, d, chunk, epochs, eta};
    run_units((long)B * H, threads, minibatch_unit, &c);
    return 0;
}

/* ==================================================================================== */
/* Conv2d preprocessing of the scan's dataset (Vision-TTT gist, item 2, "Conv2d Module":  */
/* a depthwise convolution aggregates neighbouring tokens on the 2-D grid before the scan */
/* starts; Vision-TTT review: "Conv2d-based dataset preprocessing").  Reading: the        */
/* dataset is the (K, V) pairs; each of K and V goes through its own 3x3 depthwise conv   */
/* on the Hg x Wg grid (one 3x3 filter per feature of each head, zero padding, no bias),  */
/* then the chunked scan of the section above runs on (Q, K', V').                        */
/* ==================================================================================== */

void ttt_oracle_dwconv_prep(const double* x, const double* w, double* out, int B, int H,
                            int Hg, int Wg, int d) {
    const long N = (long)Hg * Wg;
    for (long u = 0; u < (long)B * H; ++u) {
        const long h = u % H;
        const double* xu = x + u * N * d;
        for (int y = 0; y < Hg; ++y)
            for (int xx = 0; xx < Wg; ++xx)
                for (int c = 0; c < d; ++c)
                    out[u * N * d + ((long)y * Wg + xx) * d + c] =
                        dwconv_at(xu, w + (h * d + c) * 9, Hg, Wg, d, y, xx, c);
    }
}

typedef struct {
    const double *q, *k, *v, *w0, *wk, *wv;
    double* out;
    int H, Hg, Wg, d, b, direction;
    double eta;
} chunked_prep_ctx;

static void chunked_prep_unit(const void* vctx, long u) {
    const chunked_prep_ctx* c = (const chunked_prep_ctx*)vctx;
    const int d = c->d, N = c->Hg * c->Wg;
    const long h = u % c->H;
    const long tok = (long)N * d;
    double* kp = (double*)malloc(sizeof(double) * (size_t)tok);
    double* vp = (double*)malloc(sizeof(double) * (size_t)tok);
    int* idx = (int*)calloc((size_t)N, sizeof(int));
    /* K' and V' of this unit: one depthwise 3x3 filter per feature of head h */
    for (int y = 0; y < c->Hg; ++y)
        for (int x = 0; x < c->Wg; ++x)
            for (int f = 0; f < d; ++f) {
                const long at = ((long)y * c->Wg + x) * d + f;
                kp[at] = dwconv_at(c->k + u * tok, c->wk + (h * d + f) * 9, c->Hg, c->Wg, d, y, x, f);
                vp[at] = dwconv_at(c->v + u * tok, c->wv + (h * d + f) * 9, c->Hg, c->Wg, d, y, x, f);
            }
    double* o = c->out + u * tok;
    memset(o, 0, sizeof(double) * (size_t)tok);
    const double* w0 = c->w0 + h * (long)d * d;
    if (c->direction >= 0) {
        for (int t = 0; t < N; ++t) idx[t] = t;
        chunked_scan(c->q + u * tok, kp, vp, w0, idx, N, d, c->b, c->eta, o);
    }
    if (c->direction <= 0) {
        for (int t = 0; t < N; ++t) idx[t] = N - 1 - t;
        chunked_scan(c->q + u * tok, kp, vp, w0, idx, N, d, c->b, c->eta, o);
    }
    free(kp);
    free(vp);
    free(idx);
}

int ttt_oracle_linear_chunked_prep(const double* q, const double* k, const double* v,
                                   const double* w0, const double* wk, const double* wv,
                                   double* out, int B, int H, int Hg, int Wg, int d, int chunk,
                                   double eta, int direction, int threads) {
    if (B <= 0 || H <= 0 || Hg <= 0 || Wg <= 0 || d <= 0 || chunk <= 0) return 1;
    if (direction < -1 || direction > 1) return 1;
    chunked_prep_ctx c = {q, k, v, w0, wk, wv, out, H, Hg, Wg, d, chunk, direction, eta};
    run_units((long)B * H, threads, chunked_prep_unit, &c);
    return 0;
}

/* ==================================================================================== */
/* The ViT^3 TTT block around the core (ViT^3 blog, "从官方代码看…": a GLU-style main      */
/* branch and a 3x3 depthwise-conv branch, concatenated and projected back to the input  */
/* width; "TTT Block 长什么样": project the input to Q, K, V, train the inner model on     */
/* (K, V), apply it to Q).  Reading (the pages give no formulas), per image, x [N, C]:    */
/*   [Q | K | V | G] = x Wqkvg              (Wqkvg [C, 4C]; Q, K, V split into H heads)  */
/*   O_h = TTT-Linear full-batch step of head h on (Q_h, K_h, V_h) from W0[h]             */
/*   M = O * sigmoid(G)                     (GLU: a gate from the same input)             */
/*   D = 3x3 depthwise conv of x on the Hg x Wg grid (taps wc [C, 3, 3], zero padding)    */
/*   y = [M | D] Wo                         (Wo [2C, C])                                  */
/* ==================================================================================== */

typedef struct {
    const double *x, *wqkvg, *w0, *wc, *wo;
    double* y;
    int Hg, Wg, C, H;
    double eta;
} block_ctx;

static void block_unit(const void* vctx, long b) {
    const block_ctx* c = (const block_ctx*)vctx;
    const int C = c->C, H = c->H, d = C / H, N = c->Hg * c->Wg;
    const double* x = c->x + b * (long)N * C;
    double* p = (double*)malloc(sizeof(double) * (size_t)N * 4 * C);
    double* qh = (double*)malloc(sizeof(double) * (size_t)N * d);
    double* kh = (double*)malloc(sizeof(double) * (size_t)N * d);
    double* vh = (double*)malloc(sizeof(double) * (size_t)N * d);
    double* oh = (double*)malloc(sizeof(double) * (size_t)N * d);
    double* o = (double*)malloc(sizeof(double) * (size_t)N * C);
    double* z = (double*)malloc(sizeof(double) * (size_t)2 * C);
    double* gw = (double*)malloc(sizeof(double) * (size_t)d * d);
    double* ws = (double*)malloc(sizeof(double) * (size_t)d * d);
    /* projections, token by token */
    for (int t = 0; t < N; ++t)
        for (int j = 0; j < 4 * C; ++j) {
            double s = 0.0;
            for (int i = 0; i < C; ++i) s += x[(long)t * C + i] * c->wqkvg[(long)i * 4 * C + j];
            p[(long)t * 4 * C + j] = s;
        }
    /* the TTT core per head */
    for (int h = 0; h < H; ++h) {
        for (int t = 0; t < N; ++t)
            for (int e = 0; e < d; ++e) {
                qh[(long)t * d + e] = p[(long)t * 4 * C + 0 * C + h * d + e];
                kh[(long)t * d + e] = p[(long)t * 4 * C + 1 * C + h * d + e];
                vh[(long)t * d + e] = p[(long)t * 4 * C + 2 * C + h * d + e];
            }
        const double* w0 = c->w0 + (long)h * d * d;
        ttt_oracle_linear_grad(kh, vh, w0, N, d, gw);
        for (long e = 0; e < (long)d * d; ++e) ws[e] = w0[e] - c->eta * gw[e];
        linear_apply(qh, ws, N, d, oh);
        for (int t = 0; t < N; ++t)
            for (int e = 0; e < d; ++e) o[(long)t * C + h * d + e] = oh[(long)t * d + e];
    }
    /* gate, conv branch, concat, output projection, token by token */
    for (int t = 0; t < N; ++t) {
        const int py = t / c->Wg, px = t % c->Wg;
        for (int ch = 0; ch < C; ++ch) {
            const double g = p[(long)t * 4 * C + 3 * C + ch];
            z[ch] = o[(long)t * C + ch] / (1.0 + exp(-g));
            z[C + ch] = dwconv_at(x, c->wc + ch * 9, c->Hg, c->Wg, C, py, px, ch);
        }
        for (int j = 0; j < C; ++j) {
            double s = 0.0;
            for (int i = 0; i < 2 * C; ++i) s += z[i] * c->wo[(long)i * C + j];
            c->y[(b * (long)N + t) * C + j] = s;
        }
    }
    free(p);
    free(qh);
    free(kh);
    free(vh);
    free(oh);
    free(o);
    free(z);
    free(gw);
    free(ws);
}

int ttt_oracle_vit3_block(const double* x, const double* wqkvg, const double* w0, const double* wc,
                          const double* wo, double* y, int B, int Hg, int Wg, int C, int H, double eta,
                          int threads) {
    if (B <= 0 || Hg <= 0 || Wg <= 0 || C <= 0 || H <= 0 || C % H != 0) return 1;
    block_ctx c = {x, wqkvg, w0, wc, wo, y, Hg, Wg, C, H, eta};
    run_units((long)B, threads, block_unit, &c);
    return 0;
}
