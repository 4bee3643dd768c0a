/*
 * ttt.h -- C ABI of the B200 (sm_100a) Test-Time-Training layer library, libttt_b200.so.
 *
 * The layer replaces attention by one step of inner training.  Per (batch b, head h) unit,
 * with Q, K, V in R^{N x d} and an inner model F_W with initial weights W0, it forms
 *     l(W) = (1/N) sum_i 1/2 ||F_W(k_i) - v_i||^2,     W* = W0 - eta * grad l(W0),
 *     o_i  = F_{W*}(q_i).
 * Source of the operation: "ViT^3: Unlocking Test-Time Training in Vision" (techloop.online
 * blog post), section on rewriting attention as online learning (train F on (K, V), take
 * W*, output F_{W*}(Q)) and its design-study section (single epoch, full batch, inner
 * learning rate 1.0; no L1-type loss).  The squared loss with 1/N is this library's reading
 * of a point the pages leave open.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers, dense row-major in the stated layout, and
 *     16-byte aligned.  Q/K/V/out share one storage type `dtype` (TTT_F32 or TTT_BF16);
 *     inner weights are always fp32.  Accumulation is fp32.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Calls
 *     are asynchronous: they enqueue kernels and return; device-side faults surface at the
 *     caller's next synchronisation.
 *   - `workspace` is caller-owned device scratch of at least the size the matching
 *     *_workspace_bytes() query returns for the same arguments (it may be NULL when that
 *     size is 0), 16-byte aligned like the tensors (a misaligned one is TTT_ERR_INVALID_ARG).
 *     The library allocates no device memory and keeps no per-call state.
 *   - Arguments are checked on the host before anything is enqueued.  Return codes:
 *       TTT_OK, TTT_ERR_INVALID_ARG (null pointer, size <= 0, misalignment, non-finite eta,
 *       inconsistent shape), TTT_ERR_UNSUPPORTED (a size outside the supported range),
 *       TTT_ERR_WORKSPACE (workspace too small), TTT_ERR_CUDA (a launch failed).
 *   - Waits inside kernels are bounded; a wait that runs out sets a device error word that
 *     ttt_device_error() reads (TTT_ERR_TIMEOUT).
 *   - Optional outputs (w_star, ...) are fp32, exact before any bf16 rounding; pass NULL to
 *     skip them.
 */
#ifndef TTT_B200_H
#define TTT_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { TTT_F32 = 0, TTT_BF16 = 1 } ttt_dtype;

typedef enum {
    TTT_OK = 0,
    TTT_ERR_INVALID_ARG = 1,
    TTT_ERR_UNSUPPORTED = 2,
    TTT_ERR_WORKSPACE = 3,
    TTT_ERR_CUDA = 4,
    TTT_ERR_TIMEOUT = 5
} ttt_status;

/* Static English text for a status code (never NULL). */
const char* ttt_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int ttt_version(void);

/* Number of kernels this library has enqueued since it was loaded (all devices, all
 * threads).  Diagnostic: lets a caller count the device work behind a call. */
unsigned long long ttt_kernel_launch_count(void);

/* Reads and clears the device error word of the current device.  Synchronises the device.
 * Writes the raw bits to *bits (may be NULL).  Returns TTT_OK when no kernel reported a
 * problem, TTT_ERR_TIMEOUT when a bounded wait ran out, TTT_ERR_CUDA on a CUDA failure. */
int ttt_device_error(unsigned int* bits);

/* Test support for the bounded waits (no counterpart on the pages).
 * ttt_debug_set_wait_limit: the limit, in SM clock cycles, of every bounded wait in kernels
 * launched afterwards on the current device; cycles <= 0 restores the default (about one
 * second).  ttt_debug_arm_fault: arms (bits != 0) or clears (0) a simulated lost transfer on
 * the current device: with TTT_FAULT_SKIP_LOAD set, the TTT-Linear tensor-core kernel (bf16,
 * d = 64) leaves out the TMA load of each CTA's last K/V tile, so that the wait for it runs
 * out and ttt_device_error() reports TTT_ERR_TIMEOUT.  Nothing faults: the kernel gives up the
 * wait, computes on stale data and ends normally.  Both return TTT_OK or TTT_ERR_CUDA; each
 * is a synchronous copy to the device, seen by kernels that start after it. */
#define TTT_FAULT_SKIP_LOAD 0x1u
int ttt_debug_set_wait_limit(long long cycles);
int ttt_debug_arm_fault(unsigned int bits);

/* --------------------------------------------------------------------------------------
 * TTT-Linear, full batch (F_W(x) = x W; TTT abstract of Sun et al.: "hidden state a linear
 * model").  Per unit u = b*H + h:
 *     G = K^T K, C = K^T V,  W* = W0[h] - (eta/N) (G W0[h] - C),  O = Q W*.
 *   q, k, v, out : [B, H, N, d]   dtype
 *   w0           : [H, d, d]      fp32, shared across the batch
 *   w_star       : [B, H, d, d]   fp32 output, or NULL
 * Supported: any N >= 1, B*H >= 1, 1 <= d <= 128; bf16 with d in {32, 64} runs the
 * tensor-core kernel (one cluster per unit, no workspace), everything else the CUDA-core
 * kernels (workspace needed).
 * ------------------------------------------------------------------------------------ */
size_t ttt_linear_fullbatch_workspace_bytes(int B, int H, int N, int d, int dtype);
int ttt_linear_fullbatch(const void* q, const void* k, const void* v, const float* w0, void* out,
                         float* w_star, int B, int H, int N, int d, float eta, int dtype,
                         void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------------------
 * The ViT^3 TTT block around the TTT-Linear core (ViT^3 blog: the block projects its input to
 * Q, K, V, trains the inner model on (K, V) and applies it to Q -- "TTT Block 长什么样"; the
 * official code joins a GLU-style main branch and a 3x3 depthwise-conv branch, concatenates
 * them and projects back to the input width -- "从官方代码看…").  This library's reading,
 * per image with x [N, C] on the Hg x Wg grid (token index row*Wg + col):
 *     [Q | K | V | G] = x Wqkvg              (Q, K, V split into H heads of d = C/H)
 *     O = ttt_linear_fullbatch(Q, K, V, W0)  (per head, learning rate eta)
 *     y = [O * sigmoid(G) | dwconv3x3(x)] Wo  (taps wc, zero padding, no bias)
 *   x, y  : [B, Hg*Wg, C] dtype;   wqkvg : [C, 4C] dtype;   wo : [2C, C] dtype
 *   w0    : [H, d, d] fp32;        wc    : [C, 3, 3] fp32
 * bf16 with C = 64, d in {32, 64} and Wg <= 63 runs the tensor-core kernels; everything else
 * the CUDA-core kernels.  The workspace (always needed) holds Q, K, V, G and O.  Errors as for
 * the other entry points (C % H != 0 is TTT_ERR_INVALID_ARG).
 * ------------------------------------------------------------------------------------ */
size_t ttt_vit3_block_workspace_bytes(int B, int Hg, int Wg, int C, int H, int dtype);
int ttt_vit3_block(const void* x, const void* wqkvg, const float* w0, const float* wc, const void* wo, void* y,
                   int B, int Hg, int Wg, int C, int H, float eta, int dtype, void* workspace,
                   size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------------------
 * Backward of the TTT-Linear full-batch step (outer training through the inner step: the
 * ViT^3 abstract's "parallelizable computation"; the ViT^3 blog notes the official code writes
 * the closed-form gradient of the inner step by hand).  For an upstream gradient dO = dL/dO of
 * the output of ttt_linear_fullbatch, with M = Q^T dO and A = W0 M^T + M W0^T, per unit:
 *     dQ = dO W*^T,  dV = (eta/N) K M,  dK = -(eta/N)(K A - V M^T),
 *     dW0[h] = sum over the batch entries b of  M - (eta/N) G M   (W0 is shared per head)
 *   q, k, v, dout, dq, dk, dv : [B, H, N, d]   dtype (dq, dk, dv are outputs)
 *   w0 : [H, d, d] fp32;  dw0 : [H, d, d] fp32 output
 * bf16 with d = 64 runs the tensor-core kernels, everything else the CUDA-core kernels; the
 * workspace is always needed.  dW0 is summed over the batch in a fixed order (deterministic).
 * ------------------------------------------------------------------------------------ */
size_t ttt_linear_fullbatch_bwd_workspace_bytes(int B, int H, int N, int d, int dtype);
int ttt_linear_fullbatch_bwd(const void* q, const void* k, const void* v, const float* w0, const void* dout,
                             void* dq, void* dk, void* dv, float* dw0, int B, int H, int N, int d, float eta,
                             int dtype, void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------------------
 * 3x3 depthwise-conv inner model on the Hg x Wg token grid (ViT^3 blog, design study: a
 * 3x3 depthwise convolution as the visual inner module).  Per image b and channel c:
 *     F_w(X)(y, x) = sum_{a,b in 0..2} w[a][b] X(y+a-1, x+b-1)   (zero padding, no bias)
 *     g[a][b] = (1/N) sum_p r(p) K(p + (a-1, b-1)),  r = F_{w0}(K) - V,  N = Hg*Wg
 *     w* = w0[c] - eta g,  O = F_{w*}(Q)
 *   q, k, v, out : [B, Hg, Wg, C] channels-last (token index = row*Wg + col), dtype
 *   w0           : [C, 3, 3] fp32, shared across the batch
 *   w_star       : [B, C, 3, 3] fp32 output, or NULL
 * ------------------------------------------------------------------------------------ */
size_t ttt_dwconv_fullbatch_workspace_bytes(int B, int Hg, int Wg, int C, int dtype);
int ttt_dwconv_fullbatch(const void* q, const void* k, const void* v, const float* w0, void* out,
                         float* w_star, int B, int Hg, int Wg, int C, float eta, int dtype,
                         void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------------------
 * TTT-MLP, full batch (TTT abstract of Sun et al.: "hidden state a two-layer MLP"):
 *     F(x) = gelu_tanh(x W1) W2,  gelu_tanh(u) = u/2 (1 + tanh(sqrt(2/pi)(u + 0.044715 u^3)))
 * with the gradient of l taken by hand (chain rule), one full-batch step, then O = F*(Q).
 *   q, k, v, out : [B, H, N, d]   dtype
 *   w1 : [H, d, hidden] fp32;  w2 : [H, hidden, d] fp32
 *   w1_star : [B, H, d, hidden], w2_star : [B, H, hidden, d] fp32 outputs, or NULL
 * ------------------------------------------------------------------------------------ */
size_t ttt_mlp_fullbatch_workspace_bytes(int B, int H, int N, int d, int hidden, int dtype);
int ttt_mlp_fullbatch(const void* q, const void* k, const void* v, const float* w1,
                      const float* w2, void* out, float* w1_star, float* w2_star, int B, int H,
                      int N, int d, int hidden, float eta, int dtype, void* workspace,
                      size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------------------
 * Chunked bidirectional TTT-Linear (Vision-TTT gist, "Technische samenvatting": update rule
 * W_t = W_{t-1} - eta grad l(W_{t-1}; x_t), mini-batch gradient descent, forward and
 * backward scan).  Per unit, with chunks c of `chunk` consecutive tokens (N % chunk == 0):
 *     W <- W0[h];  for each chunk in order:  W <- W - (eta/chunk) K_c^T (K_c W - V_c);
 *                                            O_c = Q_c W      (W after the chunk's update)
 * run once in raster order and once in reverse raster order (both from W0); the layer
 * output is the sum of the two scans, added in fp32 and rounded once.
 *   q, k, v, out : [B, H, N, d] dtype;  w0 : [H, d, d] fp32
 * ------------------------------------------------------------------------------------ */
size_t ttt_linear_chunked_bidir_workspace_bytes(int B, int H, int N, int d, int chunk, int dtype);
int ttt_linear_chunked_bidir(const void* q, const void* k, const void* v, const float* w0,
                             void* out, int B, int H, int N, int d, int chunk, float eta,
                             int dtype, void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------------------
 * Chunked TTT-Linear scan in one direction or in both (Vision-TTT gist, "Technische
 * samenvatting": item 1 the online update, item 2 the forward and backward scan, item 3 the
 * mini-batches).  The recurrence is the one of ttt_linear_chunked_bidir above;
 *   direction = +1: raster order only, O_c = Q_c W_c (the original one-way scan)
 *   direction = -1: reverse raster order only
 *   direction =  0: both, summed (identical to ttt_linear_chunked_bidir)
 * Layouts and errors as for ttt_linear_chunked_bidir; direction outside {-1, 0, 1} is
 * TTT_ERR_INVALID_ARG.  A one-way scan on the tensor-core path needs no workspace.
 * ------------------------------------------------------------------------------------ */
size_t ttt_linear_chunked_workspace_bytes(int B, int H, int N, int d, int chunk, int direction, int dtype);
int ttt_linear_chunked(const void* q, const void* k, const void* v, const float* w0, void* out, int B, int H,
                       int N, int d, int chunk, float eta, int direction, int dtype, void* workspace,
                       size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------------------
 * Mini-batch / multi-epoch inner training of TTT-Linear, then the trained model applied to Q
 * (the inner-training options that the ViT^3 blog's design study varies -- full batch or
 * mini-batch, number of epochs -- with the per-mini-batch update of the Vision-TTT gist):
 *     W <- W0[h];  repeat `epochs` times:  for each chunk c in raster order:
 *                                            W <- W - (eta/chunk) K_c^T (K_c W - V_c)
 *     O = Q W_final   (every token sees the final weights; nothing is output per chunk)
 *   q, k, v, out : [B, H, N, d] dtype;  w0 : [H, d, d] fp32
 *   w_final      : [B, H, d, d] fp32 output, or NULL
 * chunk must divide N; epochs >= 1 (else TTT_ERR_INVALID_ARG).  chunk == N with one epoch is
 * the full-batch step and runs ttt_linear_fullbatch.  The workspace is always needed.
 * ------------------------------------------------------------------------------------ */
size_t ttt_linear_minibatch_workspace_bytes(int B, int H, int N, int d, int chunk, int epochs, int dtype);
int ttt_linear_minibatch(const void* q, const void* k, const void* v, const float* w0, void* out, float* w_final,
                         int B, int H, int N, int d, int chunk, int epochs, float eta, int dtype, void* workspace,
                         size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------------------
 * Chunked scan on a Conv2d-preprocessed dataset (Vision-TTT gist, item 2 "Conv2d Module": a
 * depthwise convolution aggregates neighbouring tokens of the 2-D grid before the scan;
 * Vision-TTT review: "Conv2d-based dataset preprocessing").  This library's reading: each of
 * K and V goes through its own 3x3 depthwise convolution on the Hg x Wg grid (one filter per
 * feature of each head, zero padding, no bias), then ttt_linear_chunked runs on (Q, K', V').
 *   q, k, v, out : [B, H, Hg*Wg, d] dtype (token index = row*Wg + col)
 *   wk, wv       : [H, d, 3, 3] fp32 filters;  w0 : [H, d, d] fp32
 * K' and V' are stored in the workspace in the input dtype; errors as for ttt_linear_chunked.
 * ------------------------------------------------------------------------------------ */
size_t ttt_linear_chunked_conv_workspace_bytes(int B, int H, int Hg, int Wg, int d, int chunk, int direction,
                                               int dtype);
int ttt_linear_chunked_conv(const void* q, const void* k, const void* v, const float* w0, const float* wk,
                            const float* wv, void* out, int B, int H, int Hg, int Wg, int d, int chunk, float eta,
                            int direction, int dtype, void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------------------------
 * ttt_linear_chunked_bidir_noalloc -- the chunked bidirectional scan above, for callers that
 * may not allocate device memory when they call (for example a runtime whose allocator is
 * owned by someone else, code that must not trigger cudaMalloc's implicit device-wide
 * synchronisation in a latency-critical loop, or an embedding that forbids allocation after
 * start-up).  It takes no workspace: its scratch is a fixed 16 MiB array inside this
 * library's device image, held by every device that loads the library until the process
 * exits.  The pages have no counterpart to this entry point; it is a service of the library.
 *   - Same arguments, layouts and results as ttt_linear_chunked_bidir, minus the workspace.
 *   - Returns TTT_ERR_WORKSPACE when ttt_linear_chunked_bidir_workspace_bytes() for these
 *     arguments exceeds ttt_linear_chunked_bidir_noalloc_max_bytes() (16 MiB: e.g. B*H*N up
 *     to 65536 for bf16, d = chunk = 64); other errors as for the workspace version.
 *   - Allocates nothing: no cudaMalloc/cudaFree or allocating library routine is called.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     for the current device; make that first call before any stream capture.
 *   - Every call shares the one array and overwrites the parts it reads before reading them
 *     (nothing needs to start at zero); calls that overlap on the GPU, on any streams of the
 *     same device, race on it and must be serialised by the caller.
 * ------------------------------------------------------------------------------------ */
int ttt_linear_chunked_bidir_noalloc(const void* q, const void* k, const void* v, const float* w0,
                                     void* out, int B, int H, int N, int d, int chunk, float eta,
                                     int dtype, void* stream);
size_t ttt_linear_chunked_bidir_noalloc_max_bytes(void);

#ifdef __cplusplus
}
#endif
#endif /* TTT_B200_H */
