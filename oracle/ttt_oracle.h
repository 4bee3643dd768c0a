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

#ifdef __cplusplus
}
#endif
#endif /* TTT_ORACLE_H */
