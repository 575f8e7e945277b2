/*
 * sparse_block.h - C ABI of the Sparse Transformer block around the
 * factorized sparse attention op (libsparse_block.so, which calls
 * libsparse_attn.so for the attention and cuBLAS and cuBLASLt for the projections).
 *
 * The block ("[논문 리뷰] Generating Long Sequences with Sparse Transformers",
 * "제안 방법", third and fourth items; the pcnews translation "Генеративное
 * моделирование с разреженными трансформерами", "Глубокое внимание"): a
 * residual block with pre-activation and layer normalisation, whose attention
 * and feed-forward parts are recomputed in the backward pass instead of
 * stored.  The pages give no formulas; the readings taken:
 *
 *   a = LN1(x);  [q | k | v] = a Wqkv;  o = attn(q, k, v)  (heads of D columns)
 *   h = x + o Wo;  f = LN2(h);  y = h + gelu(f W1) W2
 *
 * with x, h, y of shape [B, N, C], C = H * D; LN over the C channels of a
 * position with a float32 gain and bias per channel, biased variance and
 * epsilon 1e-5; gelu(u) = u Phi(u) exactly (erf form); W1: C x 4C, W2: 4C x C;
 * no projection biases; head h takes columns h*D .. h*D + D - 1 of each of q,
 * k, v and of the attention output; attn is sparse_attn_fwd with the layout
 * given and the default scale 1/sqrt(D).
 *
 * Tensors: device pointers, row-major, 16-byte aligned; activations and
 * projection weights bf16 ([in][out] for a weight: x W multiplies a row of x
 * by the weight's rows); layer-norm parameters and all parameter gradients
 * float32.  Every call is asynchronous on `stream` (a cudaStream_t, or NULL
 * for the legacy default stream) and returns an sa_status of sparse_attn.h;
 * argument errors are returned before any device work.  Calls from several
 * host threads are safe (their enqueues are serialised); calls whose GPU work
 * overlaps must not share a workspace.
 */
#ifndef SPARSE_BLOCK_H
#define SPARSE_BLOCK_H

#include <stddef.h>
#include <stdint.h>

#include "sparse_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* The block's parameters (device pointers, caller-owned). */
typedef struct sb_params {
  const float* ln1_g; /* [C] */
  const float* ln1_b; /* [C] */
  const void* w_qkv;  /* bf16 [C][3C]: columns 0..C-1 give q, C..2C-1 k, 2C..3C-1 v */
  const void* w_o;    /* bf16 [C][C] */
  const float* ln2_g; /* [C] */
  const float* ln2_b; /* [C] */
  const void* w_1;    /* bf16 [C][4C] */
  const void* w_2;    /* bf16 [4C][C] */
} sb_params;

/* Gradients of the parameters (float32 device arrays of the parameters'
 * shapes, caller-owned; overwritten, not accumulated into). */
typedef struct sb_grads {
  float* ln1_g;
  float* ln1_b;
  float* w_qkv;
  float* w_o;
  float* ln2_g;
  float* ln2_b;
  float* w_1;
  float* w_2;
} sb_grads;

/* Bytes of device workspace sparse_block_fwd / sparse_block_bwd need (the
 * activations recomputed in the backward pass, their gradients and the
 * attention's own backward workspace).  0 for an invalid shape. */
size_t sparse_block_workspace_size(int B, int N, int H, int D, const sa_layout* layout);

/*
 * sparse_block_fwd - y = block(x).  x, y: bf16 [B, N, H*D] (y must not
 * alias x, and must not overlap x or the workspace: the residual stream
 * h = x + attn(LN1(x)) is built in y before y = h + ff(LN2(h)), so after an
 * error y holds unspecified values).  D in {32, 64, 128}; layout as for
 * sparse_attn_fwd (its N).
 * workspace: at least sparse_block_workspace_size() bytes, 256-byte
 * aligned, contents on entry irrelevant, on exit unspecified.
 * Errors: SA_ERR_INVALID_ARG (null pointer, non-positive size, y == x),
 * SA_ERR_WORKSPACE (workspace null or too small), SA_ERR_UNSUPPORTED (D not
 * in {32, 64, 128}, or H*D above 6144), the errors of sparse_attn_fwd,
 * SA_ERR_CUDA when a cuBLAS or cuBLASLt call or a launch fails.
 */
int sparse_block_fwd(const void* x, const sb_params* p, void* y, int B, int N, int H, int D,
                     const sa_layout* layout, void* workspace, size_t ws_bytes, void* stream);

/*
 * sparse_block_gelu - the block's feed-forward activation on its own,
 * elementwise over n bf16 values: g = gelu(u) = u Phi(u) and, when dgelu is
 * not null, dgelu = gelu'(u) = Phi(u) + u phi(u) (Phi, phi: the standard
 * normal distribution and density).  Phi is taken from the rational
 * approximation of erfc in Abramowitz and Stegun, Handbook of Mathematical
 * Functions, eq. 7.1.26: absolute error below 7.5e-8 in Phi, so below
 * |u| 7.5e-8 in gelu (relative error grows only in the far negative tail,
 * where |gelu(u)| < 1.5e-6), before the bf16 rounding of the result.
 * u, g, dgelu: device pointers, 16-byte aligned; n a multiple of 8; g may
 * be u (in place); dgelu must be neither.  Enqueued on stream.
 * Errors: SA_ERR_INVALID_ARG (u or g null, n not a multiple of 8, a pointer
 * not 16-byte aligned, dgelu equal to u or g), SA_ERR_CUDA (launch failure).
 */
int sparse_block_gelu(const void* u, void* g, void* dgelu, size_t n, void* stream);

/*
 * sparse_block_bwd - given dy (bf16 [B, N, H*D]), the gradients of
 * sum(y * dy): dx (bf16 [B, N, H*D]) and every parameter (g, float32).
 * Only x is read from the forward pass: the whole block is recomputed from
 * it first (the recomputation of the pages), then differentiated.  dq of the
 * attention, the projection-weight gradients and the layer-norm parameter
 * gradients are float32 sums whose last bits may vary from run to run.
 * The projection-weight gradients are computed on a second stream of the
 * library's own (one a device, with its own cuBLAS handle), forked from
 * `stream` by events as their operands become ready and joined back into it
 * before the call returns, so all of the call's work is ordered before what
 * the caller enqueues on `stream` next (this fork and join can be captured
 * into a CUDA graph).
 * Errors: as sparse_block_fwd, plus those of sparse_attn_bwd.
 */
int sparse_block_bwd(const void* x, const void* dy, const sb_params* p, void* dx, const sb_grads* g,
                     int B, int N, int H, int D, const sa_layout* layout, void* workspace,
                     size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_BLOCK_H */
