/*
 * sparse_attn.h - C ABI of the B200 (sm_100a) causal factorized sparse
 * self-attention library (Sparse Transformer attention, forward and
 * backward).
 *
 * What is computed.  For one (batch b, head h) slice with queries, keys and
 * values q, k, v of shape [N, D]:
 *     S_ij = <q_i, k_j> / sqrt(D)          for (i, j) in the pattern's mask
 *     lse_i = log sum_j exp S_ij,  P = exp(S - lse),  O = P V
 * and, in the backward pass, the gradients dQ, dK, dV of sum(O * dO).
 * This is ordinary masked softmax attention ("Insights: 희소 어텐션
 * (Sparse Attention)", the attention_impl / blocksparse_attention_impl
 * paragraph), restricted to a sparse factorized mask ("OpenAI Sparse
 * Transformer", sections "Sparse Attention and Algorithmic Complexity" and
 * "Factorized Attention Patterns"; pcnews translation "Генеративное
 * моделирование с разреженными трансформерами", section "Разреженное
 * внимание").
 *
 * Masks (every mode is causal and includes j == i):
 *   SA_ALL      j <= i                                    (dense causal)
 *   SA_LOCAL    0 <= i - j < l                            (window of l)
 *   SA_STRIDED  0 <= i - j < l  or  (i - j) mod l == 0    (row + column)
 *   SA_FIXED    j <= i and ( j / l == i / l  or  j mod l >= l - c )
 *               (own l-block + the last c "summary" offsets of each block)
 *   SA_COLUMN   j <= i and (i - j) mod l == 0
 *               (the column head of SA_STRIDED run as a head of its own;
 *               its row head is SA_LOCAL)
 *   SA_BLOCK    j <= i and j / l == i / l
 *               (the own-block head of SA_FIXED run as a head of its own)
 *   SA_BLOCKS   j <= i and block (i / b, j / b) is in a caller's block mask
 *               (built with sparse_attn_layout_blocks: the sparsity pattern
 *               given as a mask over blocks, the SparseAttention(q, k, v,
 *               mask) form of "Insights: 희소 어텐션 (Sparse Attention)")
 * SA_COLUMN and SA_BLOCK are the two-head form of the factorized patterns:
 * the two parts of a pattern in separate heads, each with its own softmax
 * ("OpenAI Sparse Transformer", "Factorized Attention Patterns"; pcnews
 * translation, "Разреженное внимание").
 *
 * The backward pass recomputes P from the saved lse and never stores an
 * N x N matrix, the memory-saving recomputation of "Generating Long
 * Sequences with Sparse Transformers" (ABSTRACT, item b) and of the pcnews
 * translation, section "Глубокое внимание".
 *
 * Tensor conventions (all calls):
 *   q, k, v, o, dO, dq, dk, dv : bfloat16, [B, H, N, D] contiguous (row
 *       major, D fastest), device pointers, 16-byte aligned, owned by the
 *       caller.  bfloat16 values are passed as raw 16-bit patterns.
 *   lse : float32 [B, H, N], natural logarithm, device pointer.
 *   D   : 32, 64 or 128.  The softmax scale is 1/sqrt(D) in the plain entry
 *         points; sparse_attn_fwd_ex / sparse_attn_bwd_ex take it explicitly.
 *   stream : a cudaStream_t passed as void*; NULL means the legacy default
 *       stream.  Every compute call only enqueues work on that stream and
 *       returns; none synchronises except sparse_attn_status().
 * Errors: every int-returning call returns SA_OK (0) or one of the
 * sa_status codes below; sparse_attn_strerror() names them.  Argument
 * errors are detected on the host before anything is enqueued.
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sa_layout sa_layout; /* opaque, owned by the library */

enum sa_pattern {
  SA_ALL = 0,
  SA_LOCAL = 1,
  SA_STRIDED = 2,
  SA_FIXED = 3,
  SA_COLUMN = 4,
  SA_BLOCK = 5,
  SA_BLOCKS = 6
};

/* Views of a pattern.  Each view is dense in its own relabelled order:
 *   SA_VIEW_NATURAL : natural order, queries and keys (every pattern but
 *       SA_COLUMN).
 *   SA_VIEW_COLUMN  : SA_STRIDED and SA_COLUMN.  Positions relabelled
 *       column-major, t(p) = (p mod l) * R + p / l with R = N / l; holds the
 *       strictly earlier positions of the same column (attending along a
 *       column is attending along a row of the transposed 2-D array: pcnews
 *       translation, "Разреженное внимание"), and for SA_COLUMN, which has
 *       no natural view, the position itself too.
 *   SA_VIEW_SUMMARY : fixed only.  Queries natural; keys are the summary
 *       positions j mod l >= l - c numbered consecutively,
 *       sigma(j) = (j / l) * c + (j mod l - (l - c)); holds the summary keys
 *       of strictly earlier blocks.
 * OR SA_VIEW_TRANSPOSED into a view id to export the key-block-major table
 * of that view (used by the backward pass). */
enum sa_view {
  SA_VIEW_NATURAL = 0,
  SA_VIEW_COLUMN = 1,
  SA_VIEW_SUMMARY = 2,
  SA_VIEW_TRANSPOSED = 4
};

enum sa_status {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad enum   */
  SA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (D, divisibility) */
  SA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed           */
  SA_ERR_LUT = 4,          /* layout does not match the call's shape      */
  SA_ERR_TIMEOUT = 5,      /* a device-side wait gave up (status word)    */
  SA_ERR_WORKSPACE = 6     /* workspace missing or too small              */
};

/* Block look-up table kinds. */
enum sa_block_kind { SA_BLOCK_FULL = 0, SA_BLOCK_PARTIAL = 1 };

/*
 * sparse_attn_layout - build the block layout of a pattern.
 *
 * The block-sparse kernels of the pages slice queries and keys into blocks
 * ("OpenAI Sparse Transformer", "Implementation and Limitations"; pcnews
 * translation, "Релиз кода"; the SparseAttention class of the "Insights"
 * page reshapes its inputs to the block size).  For every view of the
 * pattern this builds, on the host, a CSR table over query blocks of
 * `block` positions listing the key blocks that hold part of the mask, in
 * ascending order, each marked FULL (every element in the mask) or PARTIAL,
 * plus its key-block-major transpose, and the coarser tile tables the
 * kernels run on.  Device copies are made on the first compute call on each
 * device (or by sparse_attn_layout_upload).
 *
 * Arguments: pattern (sa_pattern); N >= 1 sequence length; l >= 1 row
 * length / window (ignored for SA_ALL); c summary columns, 1 <= c <= l
 * (SA_FIXED only, ignored otherwise); block >= 1 with N % block == 0.
 * SA_STRIDED, SA_FIXED and SA_COLUMN need N % l == 0.  *out receives a layout the
 * caller releases with sparse_attn_layout_free.
 * Errors: SA_ERR_INVALID_ARG (bad pattern, sizes, null out),
 * SA_ERR_UNSUPPORTED (N % block or N % l not zero).
 */
int sparse_attn_layout(int pattern, int N, int l, int c, int block, sa_layout** out);

/*
 * sparse_attn_layout_blocks - a layout (pattern SA_BLOCKS) from a caller's
 * block mask: the sparsity pattern given as a mask over blocks (the
 * SparseAttention(q, k, v, mask) form of "Insights: 희소 어텐션 (Sparse
 * Attention)").  row_ptr [N/block + 1] and col_idx (host memory, read
 * during the call only) list, per query block r, the key blocks s in the
 * mask, ascending, with 0 <= s <= r and the diagonal block s = r last (so
 * no row is empty).  Element (i, j) attends when its block is listed and
 * j <= i.  block must divide N and be a multiple of 128 (every kernel tile
 * then lies inside one block) or one of 16, 32, 64 (a kernel tile then
 * holds several blocks and masks the unlisted ones element by element).
 * Errors: SA_ERR_INVALID_ARG (null pointer, N < 1, a row that is empty,
 * unsorted, above the diagonal or without its diagonal block),
 * SA_ERR_UNSUPPORTED (another block size, N % block not zero).
 */
int sparse_attn_layout_blocks(int N, int block, const int32_t* row_ptr, const int32_t* col_idx,
                              sa_layout** out);

/*
 * sparse_attn_layout_export - host copy of one view's block table.
 * view: an sa_view id, optionally OR SA_VIEW_TRANSPOSED.  Any of row_ptr
 * (n_rows + 1 entries), col_idx, kind (nnzb entries each) may be NULL; the
 * sizes are always written to *n_rows and *nnzb (both required).
 * A view the pattern does not have exports as zero rows.
 * Errors: SA_ERR_INVALID_ARG.
 */
int sparse_attn_layout_export(const sa_layout* layout, int view, int32_t* row_ptr,
                              int32_t* col_idx, uint8_t* kind, int* n_rows, int* nnzb);

/* Pattern parameters stored in a layout (any output pointer may be NULL). */
int sparse_attn_layout_info(const sa_layout* layout, int* pattern, int* N, int* l, int* c,
                            int* block);

/* Copy the layout's tables to the current device now, on `stream`
 * (otherwise the first compute call does it).  Call before any stream
 * capture.  Errors: SA_ERR_INVALID_ARG, SA_ERR_CUDA. */
int sparse_attn_layout_upload(const sa_layout* layout, void* stream);

/* Release a layout and its device copies (synchronises the device). */
void sparse_attn_layout_free(sa_layout* layout);

/*
 * sparse_attn_fwd - forward pass.  Writes o [B,H,N,D] (bf16) and lse
 * [B,H,N] (fp32, natural log).  For SA_STRIDED the column view runs first
 * and its partial result is merged exactly (log-sum-exp) into the natural
 * view's; SA_COLUMN runs the column view alone.  layout must have been
 * built for this N.
 * Errors: SA_ERR_INVALID_ARG (null pointer, B/H < 1), SA_ERR_LUT (layout N
 * differs), SA_ERR_UNSUPPORTED (D not 32/64/128, column geometry the
 * kernels do not tile: R = N/l must be a multiple of 8 and divide or be
 * divisible by 128), SA_ERR_CUDA.
 */
int sparse_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int H, int N, int D, const sa_layout* layout, void* stream);

/*
 * sparse_attn_fwd_ex - sparse_attn_fwd with the softmax scale given: scores
 * are scale * q.k (sparse_attn_fwd uses 1/sqrt(D); the pages do not fix the
 * scale, see "Insights: 희소 어텐션 (Sparse Attention)", the attention_impl
 * paragraph).  lse = log sum_j exp(scale * q_i.k_j).  scale must be finite
 * and > 0, else SA_ERR_INVALID_ARG (returned before any launch); the other
 * arguments and errors are those of sparse_attn_fwd.
 */
int sparse_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int H, int N, int D, float scale, const sa_layout* layout, void* stream);

/* Bytes of device workspace sparse_attn_bwd needs for this shape. */
size_t sparse_attn_bwd_workspace_size(int B, int H, int N, int D, const sa_layout* layout);

/*
 * sparse_attn_bwd - backward pass with recomputation.  Inputs q, k, v, o,
 * lse (as written by sparse_attn_fwd) and dO; outputs dq, dk, dv (bf16).
 * workspace: caller-owned device memory of at least
 * sparse_attn_bwd_workspace_size() bytes, 256-byte aligned; its contents on
 * entry do not matter and on exit are unspecified.  dq accumulates in
 * float32 by bulk reduce-adds in arrival order where several key tiles of a
 * pass meet a query row, so its last bits may vary from run to run; dk and
 * dv are deterministic.
 * Errors: as sparse_attn_fwd, plus SA_ERR_WORKSPACE.
 */
int sparse_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                    const float* lse, const void* dO, void* dq, void* dk, void* dv, int B, int H,
                    int N, int D, const sa_layout* layout, void* workspace, size_t ws_bytes,
                    void* stream);

/*
 * sparse_attn_bwd_ex - sparse_attn_bwd with the softmax scale given (the
 * scale the forward pass that produced o and lse used; dQ and dK carry the
 * factor scale).  scale must be finite and > 0, else SA_ERR_INVALID_ARG
 * (returned before any launch); the other arguments and errors are those of
 * sparse_attn_bwd.
 */
int sparse_attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                       const float* lse, const void* dO, void* dq, void* dk, void* dv, int B,
                       int H, int N, int D, float scale, const sa_layout* layout, void* workspace,
                       size_t ws_bytes, void* stream);

/*
 * sparse_attn_bwd_noalloc - the backward pass for callers that cannot
 * allocate device memory.  (Library-specific; the pages have no counterpart.)
 *
 * Some callers may not call cudaMalloc at all: for example a host framework
 * that has handed every byte of device memory to its own pool and forbids
 * outside allocations, or an application with a rule against device
 * allocation after start-up.  They cannot supply the workspace that
 * sparse_attn_bwd needs.  This entry point takes the same arguments minus the
 * workspace and uses instead a scratch array compiled into the library: a
 * file-scope __device__ array of SA_NOALLOC_SCRATCH_BYTES bytes, which every
 * GPU that loads the library holds until the process exits.  That memory is
 * taken when the library's device code is loaded on a device (with lazy
 * module loading, at the first launch of any of its kernels there), so a
 * caller's device-memory budget must count it from then on.
 *
 * Limits and behaviour (the checks run in this order, before any device
 * work: pointer and shape arguments, then the size, then the layout):
 *  - shapes whose sparse_attn_bwd_workspace_size() exceeds
 *    SA_NOALLOC_SCRATCH_BYTES are rejected with SA_ERR_WORKSPACE;
 *  - it calls no cudaMalloc, cudaFree or other allocating routine, so the
 *    layout's tables must already be on the current device (call
 *    sparse_attn_layout_upload, or any other compute call with this layout,
 *    on this device first); otherwise it returns SA_ERR_INVALID_ARG;
 *  - the first call on a device looks up the device address of the scratch
 *    array (cudaGetSymbolAddress) once for that device; make that first call
 *    before any stream capture;
 *  - every call on a device shares the one array, which keeps whatever the
 *    last call left in it.  The kernels set everything they read from it
 *    (the dQ accumulator is cleared by the preprocess kernel or wholly
 *    overwritten by the first pass that meets it), so no clearing
 *    is needed between calls, but calls whose GPU work overlaps (different
 *    streams, or different host threads) race on the array and give wrong
 *    results: order them on one stream or with events.
 * Results equal those of sparse_attn_bwd (dq up to the run-to-run rounding of
 * its fp32 reductions, which add in arrival order).  Errors: as
 * sparse_attn_bwd.
 */
#define SA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
int sparse_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dO, void* dq, void* dk, void* dv,
                            int B, int H, int N, int D, const sa_layout* layout, void* stream);

/*
 * sparse_attn_status - synchronise `stream`, then read and clear the
 * current device's status word.  Kernels never trap: a device-side wait
 * that gives up (about two seconds without progress) records
 * SA_ERR_TIMEOUT there and the kernel drains and returns.  Returns SA_OK,
 * SA_ERR_TIMEOUT or SA_ERR_CUDA (a pending CUDA error).
 */
int sparse_attn_status(void* stream);

/* Static, human-readable name of a status code. */
const char* sparse_attn_strerror(int status);

/*
 * Instrumentation for benchmarks (off by default; no effect on results).
 * sparse_attn_timing_enable(1) brackets every kernel launch with CUDA
 * events on its stream; sparse_attn_timing_read(i, ...) returns, for kind i
 * in [0, sparse_attn_kernel_kinds()), its name ("<kernel>.<pattern>", one
 * kind per kernel and pattern), the summed elapsed milliseconds of
 * completed launches and their count (it synchronises the events).  sparse_attn_timing_reset() clears the sums.
 * sparse_attn_launch_count() counts every kernel this library has launched
 * since load (timing on or off).
 */
int sparse_attn_kernel_kinds(void);
int sparse_attn_timing_enable(int on);
int sparse_attn_timing_reset(void);
int sparse_attn_timing_read(int kind, const char** name, double* total_ms, long long* launches);
long long sparse_attn_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */
