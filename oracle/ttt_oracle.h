/*
 * ttt_oracle.h -- prototypes of the fp64 CPU oracle (test infrastructure only; see
 * ttt_oracle.c for the definitions it follows).  All arrays are double, row-major:
 *   q, k, v, out : [B, H, N, d] (linear, MLP, chunked) or [B, Hg, Wg, C] (conv)
 *   w0           : [H, d, d] (linear, chunked), [C, 3, 3] (conv)
 *   w1, w2       : [H, d, h] and [H, h, d] (MLP)
 *   w_star       : [B, H, d, d] / [B, C, 3, 3] / [B, H, d, h] + [B, H, h, d], or NULL
 * Every *_fullbatch / *_chunked function returns 0 on success, 1 on a bad argument.
 */
#ifndef TTT_ORACLE_H
#define TTT_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

double ttt_oracle_linear_loss(const double* k, const double* v, const double* w, int N, int d);
void ttt_oracle_linear_grad(const double* k, const double* v, const double* w, int N, int d,
                            double* g);
int ttt_oracle_linear_fullbatch(const double* q, const double* k, const double* v,
                                const double* w0, double* out, double* w_star, int B, int H,
                                int N, int d, double eta, int threads);

double ttt_oracle_dwconv_loss(const double* k, const double* v, const double* w, int Hg,
                              int Wg, int C);
void ttt_oracle_dwconv_grad(const double* k, const double* v, const double* w, int Hg, int Wg,
                            int C, double* g);
int ttt_oracle_dwconv_fullbatch(const double* q, const double* k, const double* v,
                                const double* w0, double* out, double* w_star, int B, int Hg,
                                int Wg, int C, double eta, int threads);

double ttt_oracle_gelu_tanh(double u);
double ttt_oracle_gelu_tanh_grad(double u);
double ttt_oracle_mlp_loss(const double* k, const double* v, const double* w1,
                           const double* w2, int N, int d, int h);
void ttt_oracle_mlp_grad(const double* k, const double* v, const double* w1, const double* w2,
                         int N, int d, int h, double* g1, double* g2);
int ttt_oracle_mlp_fullbatch(const double* q, const double* k, const double* v,
                             const double* w1, const double* w2, double* out, double* w1_star,
                             double* w2_star, int B, int H, int N, int d, int h, double eta,
                             int threads);

int ttt_oracle_linear_chunked(const double* q, const double* k, const double* v,
                              const double* w0, double* out, int B, int H, int N, int d,
                              int chunk, double eta, int direction, int threads);

/* backward of the full-batch TTT-Linear step: dout [B,H,N,d] -> dq, dk, dv [B,H,N,d],
 * dw0 [H,d,d] (summed over the batch) */
int ttt_oracle_linear_fullbatch_bwd(const double* q, const double* k, const double* v,
                                    const double* w0, const double* dout, double* dq,
                                    double* dk, double* dv, double* dw0, int B, int H, int N,
                                    int d, double eta, int threads);

/* E epochs of mini-batch inner training (chunks of `chunk` tokens, raster order), then
 * out = Q W_final; w_final [B,H,d,d] or NULL */
int ttt_oracle_linear_minibatch(const double* q, const double* k, const double* v,
                                const double* w0, double* out, double* w_final, int B, int H,
                                int N, int d, int chunk, int epochs, double eta, int threads);

/* 3x3 depthwise conv of x [B,H,Hg*Wg,d] with taps w [H,d,3,3] (zero padding) */
void ttt_oracle_dwconv_prep(const double* x, const double* w, double* out, int B, int H,
                            int Hg, int Wg, int d);

/* chunked scan on (Q, dwconv(K; wk), dwconv(V; wv)); wk, wv [H,d,3,3] */
int ttt_oracle_linear_chunked_prep(const double* q, const double* k, const double* v,
                                   const double* w0, const double* wk, const double* wv,
                                   double* out, int B, int H, int Hg, int Wg, int d, int chunk,
                                   double eta, int direction, int threads);

/* ViT^3 TTT block: x [B, Hg*Wg, C] -> y [B, Hg*Wg, C]; wqkvg [C, 4C], w0 [H, C/H, C/H],
 * wc [C, 3, 3], wo [2C, C] */
int ttt_oracle_vit3_block(const double* x, const double* wqkvg, const double* w0, const double* wc,
                          const double* wo, double* y, int B, int Hg, int Wg, int C, int H, double eta,
                          int threads);

#ifdef __cplusplus
}
#endif
#endif /* TTT_ORACLE_H */
