/*
 * ks.h -- C ABI of the B200 (sm_100a) library for multiplication by
 * Kronecker-sparse (KS) matrices.
 *
 * The operation (taxoreview.com page on Kronecker-sparse matrix
 * multiplication, first abstract: KS supports are Kronecker products of
 * identity and all-ones blocks; butterfly and Monarch matrices are products of
 * KS factors).  Read with the textbook Kronecker index order, a KS factor of
 * pattern (a, b, c, d) is the (a*b*d) x (a*c*d) matrix K with support
 * I_a (x) 1_{b x c} (x) I_d,
 *
 *     K[i*b*d + k*d + l][i*c*d + j*d + l] = values[i][l][k][j],
 *     i < a, k < b, j < c, l < d,
 *
 * and the library computes, for a batch of `batch` rows,
 *
 *     Y[n][i*b*d + k*d + l] = sum_{j<c} values[i][l][k][j] * X[n][i*c*d + j*d + l],
 *
 * i.e. Y = X * K^T, without ever forming K and without permutation kernels.
 *
 * Conventions shared by every entry point
 *   - Pointers named X, values, factors[t], Y are DEVICE pointers (memory of
 *     the current CUDA device), owned by the caller.  The library keeps none
 *     of them after the call returns and frees nothing it did not allocate.
 *   - X is batch x (a*c*d) row-major; Y is batch x (a*b*d) row-major;
 *     values is the contiguous array values[a][d][b][c].
 *   - X, values and Y share one storage type: fp32 for KS_F32 and KS_TF32,
 *     bf16 for KS_BF16 (Y is written in bf16, rounded to nearest even from an
 *     fp32 accumulator).  KS_TF32 reads and writes fp32 buffers; where the
 *     tensor-core kernel takes the pattern (see KS_TF32 below) the products
 *     use TF32 operands with fp32 accumulation, elsewhere they are full fp32.
 *     TF32 is never chosen silently for KS_F32.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call is asynchronous on that stream; the return value reports only
 *     errors found before or at launch.  Errors found on the device (a bounded
 *     wait that gave up) are reported by ks_sync_status().
 *   - Calls run on the calling thread's current CUDA device; device buffers
 *     and the stream must belong to it.  The library's per-device state
 *     (workspace pool, status word, helper streams) is kept per device, so a
 *     process may drive several GPUs by switching the current device.
 *   - Y must not overlap X or values (KS_ERR_INVALID_ARG).
 *   - batch == 0 is a no-op returning KS_OK.  Negative or zero pattern
 *     entries, negative batch, or sizes whose element counts overflow int64
 *     return KS_ERR_INVALID_ARG.  Any pointer alignment is accepted (fp32
 *     needs 4-byte, bf16 2-byte alignment at least, else KS_ERR_MISALIGNED);
 *     16-byte aligned pointers and row widths take the vectorised kernels.
 *   - No exception crosses this interface.  All calls are thread-safe; the
 *     message of the last failing call is kept per host thread.
 */
#ifndef KS_B200_KS_H
#define KS_B200_KS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Storage / arithmetic type of X, values and Y. */
/* KS_TF32 and KS_BF16 run on the tcgen05 tensor cores when the pattern fits
 * the tensor-core kernel: d in {1, 2, 4} or a multiple of 8; c a multiple of
 * 8 (TF32) or 16 (BF16); b a multiple of 16; b*c > 64; X, values and Y
 * 16-byte aligned.  Other patterns run on CUDA cores with fp32 arithmetic
 * (at least the accuracy of the tensor-core path). */
typedef enum ks_dtype {
    KS_F32 = 0,  /* fp32 storage, fp32 FMA arithmetic (CUDA cores)                 */
    KS_TF32 = 1, /* fp32 storage, TF32 tensor-core products, fp32 accumulate       */
    KS_BF16 = 2  /* bf16 storage, bf16 tensor-core products, fp32 accumulate       */
} ks_dtype;

typedef enum ks_status {
    KS_OK = 0,
    KS_ERR_INVALID_ARG = 1, /* bad pattern, batch, dtype, pointer or overlap          */
    KS_ERR_MISALIGNED = 2,  /* pointer not aligned to its element size                */
    KS_ERR_UNSUPPORTED = 3, /* variant forced on a pattern it cannot run              */
    KS_ERR_ALLOC = 4,       /* workspace allocation failed                            */
    KS_ERR_CUDA = 5,        /* a CUDA runtime call failed; see ks_last_error()        */
    KS_ERR_TIMEOUT = 6      /* a bounded device-side wait gave up (ks_sync_status)    */
} ks_status;

/* Kernel families.  KS_VARIANT_AUTO lets the library's pattern heuristic
 * choose; the others force one family (for tests and measurements). */
typedef enum ks_variant {
    KS_VARIANT_AUTO = 0,
    KS_VARIANT_STREAM = 1, /* bandwidth kernel: each thread reads its c inputs
                              directly; any pattern, meant for b, c <= 8      */
    KS_VARIANT_FMA = 2,    /* output-stationary CUDA-core gather-GEMM          */
    KS_VARIANT_TC = 3      /* tcgen05 tensor-core block-GEMM (TF32 / BF16)     */
} ks_variant;

/* Pointwise activation of a fused epilogue (ks_matmul_ep, ks_chain_ep).
 * GELU is z * Phi(z), Phi the standard normal distribution function, either
 * exactly through erf or in the usual tanh form
 * z * (1 + tanh(sqrt(2/pi) * (z + 0.044715 z^3))) / 2. */
typedef enum ks_activation {
    KS_ACT_NONE = 0,
    KS_ACT_RELU = 1,      /* max(z, 0)                        */
    KS_ACT_GELU_TANH = 2, /* GELU, tanh form (CUDA tanhf)     */
    KS_ACT_GELU_ERF = 3   /* GELU, erf form (CUDA erff)       */
} ks_activation;

/* One factor's pattern: K is (a*b*d) x (a*c*d) with support I_a (x) 1_{b x c} (x) I_d. */
typedef struct ks_pattern {
    int64_t a, b, c, d;
} ks_pattern;

/* Y = X * K^T for one KS factor (see the top of this file for the layout).
 * dtype is a ks_dtype; stream a cudaStream_t.  The pattern heuristic picks the
 * kernel.
 *
 * Workspace: for KS_F32 (and KS_TF32 patterns on CUDA cores) with d % 8 == 0,
 * b % 4 == 0, at least 2^30 flop (2*batch*a*b*c*d) and values of at most
 * 64 MiB, the product first writes a copy of the values transposed per block
 * into a stream-ordered workspace (a*b*c*d floats) from the library's memory
 * pool (see ks_chain) and frees it on the stream after the kernel; if that
 * allocation fails the values are read in place and the result is the same.
 * Every other product allocates nothing.  ks_chain_noalloc never takes this
 * workspace. */
ks_status ks_matmul(const void *X, const void *values, int64_t a, int64_t b,
                    int64_t c, int64_t d, int64_t batch, void *Y, int dtype,
                    void *stream);

/* ks_matmul for a batch that lives in HOST memory: X (batch x a*c*d),
 * values and Y (batch x a*b*d) are HOST pointers, laid out as for ks_matmul.
 * The library copies the values to the device once and streams the rows
 * through in chunks (1 to 32, more for larger batches, each a multiple of
 * 128 rows):
 * the copy of chunk k+1 to the device, the product of chunk k and the copy of
 * chunk k-1 back to the host run at the same time, on three streams the
 * library keeps per device, ordered after earlier work on `stream`; `stream`
 * waits for the whole call, which is asynchronous like every entry point
 * (synchronise `stream` before reading Y or reusing X).  Page-locked host
 * memory (cudaHostAlloc / cudaHostRegister) lets the copies overlap; pageable
 * memory gives the same result without the overlap.  The device buffers (the
 * values and two chunks of X and of Y) come from the library's pool, stream-
 * ordered on `stream` (KS_ERR_ALLOC if that fails).  The product of each chunk
 * is the one ks_matmul picks. */
ks_status ks_matmul_host(const void *X, const void *values, int64_t a, int64_t b,
                         int64_t c, int64_t d, int64_t batch, void *Y, int dtype,
                         void *stream);

/* ks_matmul with a fused epilogue (the MLP shapes' bias and activation):
 *     Y[n][col] = act(sum_j ... + bias[col]),  col = i*b*d + k*d + l,
 * computed on the fp32 accumulator before the single rounding to the storage
 * dtype, inside the same kernel (no extra pass over Y).  bias is a DEVICE
 * array of a*b*d elements of the storage dtype, or NULL for none; activation
 * is a ks_activation (other values: KS_ERR_INVALID_ARG).  bias must not
 * overlap Y.  variant is a ks_variant as for ks_matmul_variant.  With bias
 * NULL, KS_ACT_NONE and KS_VARIANT_AUTO this is ks_matmul.  The tensor-core
 * kernel (KS_TF32, KS_BF16) takes a bias only if it is 16-byte aligned (else
 * the CUDA-core kernel runs) and computes the tanh form of GELU with the
 * hardware tanh approximation (relative error about 2^-11, far inside the
 * TF32 and bf16 tolerances); KS_F32 products evaluate it as z / (1 + 2^s),
 * s = -2 log2(e) sqrt(2/pi) (z + 0.044715 z^3), through the PTX ex2.approx
 * and rcp.approx instructions (a few fp32 ulps). */
ks_status ks_matmul_ep(const void *X, const void *values, int64_t a, int64_t b,
                       int64_t c, int64_t d, int64_t batch, void *Y, int dtype,
                       const void *bias, int activation, int variant,
                       void *stream);

/* ks_matmul with the kernel family forced (a ks_variant).  Returns
 * KS_ERR_UNSUPPORTED if that family cannot run this pattern / dtype /
 * alignment (e.g. KS_VARIANT_TC with dtype KS_F32). */
ks_status ks_matmul_variant(const void *X, const void *values, int64_t a,
                            int64_t b, int64_t c, int64_t d, int64_t batch,
                            void *Y, int dtype, int variant, void *stream);

/* Input gradient of Y = X * K^T (training the page's KSLinear layer):
 *     dX = dY * K,  dX[n][i*c*d + j*d + l] = sum_{k<b} values[i][l][k][j] * dY[n][i*b*d + k*d + l].
 * dY is batch x (a*b*d), dX is batch x (a*c*d), values as for ks_matmul; all
 * DEVICE pointers of one dtype.  dX is overwritten and must not overlap dY or
 * values (KS_ERR_INVALID_ARG).  This is the KS product of pattern (a, c, b, d)
 * with every block transposed: the library transposes the values into a
 * stream-ordered workspace from its pool (a*b*c*d elements, freed before
 * return; KS_ERR_ALLOC if that fails) and runs the kernel ks_matmul picks for
 * (a, c, b, d).  batch == 0 is a no-op. */
ks_status ks_matmul_dx(const void *dY, const void *values, int64_t a, int64_t b,
                       int64_t c, int64_t d, int64_t batch, void *dX, int dtype,
                       void *stream);

/* Values gradient of Y = X * K^T:
 *     dV[i][l][k][j] = sum_{n<batch} dY[n][i*b*d + k*d + l] * X[n][i*c*d + j*d + l],
 * written (not accumulated) in the values layout [a][d][b][c].  dY is
 * batch x (a*b*d), X batch x (a*c*d); DEVICE pointers of one dtype, dV must
 * not overlap dY or X.  Sums are fp32 over ranges of rows: on CUDA cores in
 * row order, or, for bf16 with d % 8 == 0, c % 16 == 0 up to 64, b >= 128 and
 * 16-byte-aligned dY and X, on the tensor cores in steps of 16 rows.  The
 * partial sums of the ranges (a stream-ordered fp32 workspace from the
 * library's pool, at most 256 MiB; KS_ERR_ALLOC if it cannot be had) are added
 * in range order, so the result is deterministic; bf16 dV is rounded once at
 * the end.  batch == 0 writes zeros. */
ks_status ks_matmul_dv(const void *dY, const void *X, int64_t a, int64_t b,
                       int64_t c, int64_t d, int64_t batch, void *dV, int dtype,
                       void *stream);

/* Bias gradient of the page's KSLinear layer, y = x K^T + bias:
 *     db[col] = sum_{n<batch} dY[n][col],  col < width.
 * dY is batch x width (DEVICE, row-major), db width elements (DEVICE), one
 * dtype; db must not overlap dY.  Sums are fp32, over row ranges in row order,
 * the ranges' partial sums (a stream-ordered fp32 workspace from the
 * library's pool, KS_ERR_ALLOC if it cannot be had) added in range order: the
 * result is deterministic; bf16 db is rounded once.  batch == 0 writes zeros. */
ks_status ks_bias_grad(const void *dY, int64_t batch, int64_t width, void *db, int dtype, void *stream);

/* What KS_VARIANT_AUTO would run for this problem, written to *variant
 * (a ks_variant).  Host-only: touches no device. */
ks_status ks_plan(int64_t a, int64_t b, int64_t c, int64_t d, int64_t batch,
                  int dtype, int *variant);

/* A chain of KS factors applied in order, factor 0 first:
 *     Y = X * (K_{n-1} ... K_1 K_0)^T.
 * factors is a HOST array of n_factors DEVICE pointers, factor t holding
 * values[a_t][d_t][b_t][c_t]; patterns is a HOST array of n_factors patterns.
 * Widths must chain: a_t*b_t*d_t == a_{t+1}*c_{t+1}*d_{t+1}, else
 * KS_ERR_INVALID_ARG.  X is batch x (a_0*c_0*d_0), Y is
 * batch x (a_{n-1}*b_{n-1}*d_{n-1}).  Intermediates (in the chain's storage
 * dtype) live in two workspace buffers allocated stream-ordered from a memory
 * pool the library owns on each device (cudaMallocFromPoolAsync) and freed to
 * it on the same stream before return (KS_ERR_ALLOC if the allocation fails).
 * The pool keeps freed memory for later calls: the device memory it holds
 * grows to the largest workspace one call has used and stays reserved until
 * the process exits.  Each factor runs the kernel the pattern heuristic
 * picks, except for the chains ks_chain_ex fuses (see there). */
ks_status ks_chain(const void *X, const void *const *factors,
                   const ks_pattern *patterns, int n_factors, int64_t batch,
                   void *Y, int dtype, void *stream);

/* Flags of ks_chain_ex. */
typedef enum ks_chain_flags {
    KS_CHAIN_UNFUSED = 1 /* apply every factor with its own kernel, never a fused one */
} ks_chain_flags;

/* ks_chain with flags (a bitwise OR of ks_chain_flags; other bits:
 * KS_ERR_INVALID_ARG).  ks_chain(...) is ks_chain_ex(..., 0, stream).
 *
 * Fusion: the twelve-factor 4096-wide butterfly chain, factors
 * (2^t, 2, 2, 2^(11-t)) for t = 0..11 in that order (the square butterfly
 * of size 4096, factor t mixing index bit 11 - t), runs as one kernel that
 * reads X once and writes Y once, keeps intermediates in fp32 (also for bf16
 * chains, which then round only Y) and allocates nothing.  It needs Y
 * 16-byte aligned and the factors 16-byte (fp32) or 8-byte (bf16) aligned;
 * otherwise, or with KS_CHAIN_UNFUSED, the chain runs factor by factor as
 * described for ks_chain.  Y must not overlap X or a factor. */
ks_status ks_chain_ex(const void *X, const void *const *factors,
                      const ks_pattern *patterns, int n_factors, int64_t batch,
                      void *Y, int dtype, int flags, void *stream);

/* ks_chain_ex with a fused epilogue on the last factor: Y = act(X (K_{n-1}
 * ... K_0)^T + bias), bias of a_{n-1}*b_{n-1}*d_{n-1} elements or NULL (as in
 * ks_matmul_ep).  A Monarch-style layer (two KS factors, then bias and
 * activation) is one call.  With an epilogue the butterfly chain is not
 * fused; its factors run one by one, the last with the epilogue. */
ks_status ks_chain_ep(const void *X, const void *const *factors,
                      const ks_pattern *patterns, int n_factors, int64_t batch,
                      void *Y, int dtype, int flags, const void *bias,
                      int activation, void *stream);

/* ks_chain without any device allocation (the paper has no counterpart: this
 * entry point serves callers that must not allocate).  Callers whose device
 * memory is owned by another allocator, such as a framework's caching pool, or
 * who run latency-critical loops where an allocation is not allowed, cannot
 * let ks_chain allocate its intermediates.  This variant keeps them in one
 * fixed array inside the library instead: 32 MiB per device, reserved on every
 * GPU that loads the library and held until the process exits, split into two
 * intermediates of at most 16 MiB each.
 *
 * Arguments, layouts and the result are exactly those of ks_chain.  A chain
 * whose intermediate (batch x intermediate width x element size) exceeds
 * 16 MiB is rejected with KS_ERR_INVALID_ARG before anything runs.  The
 * first call on a device looks up that device's address of the array
 * (cudaGetSymbolAddress, with the device current); make that first call before
 * any stream capture.  Nothing is cleared between calls: each intermediate is
 * written in full before it is read.  All calls share the one array, so calls
 * whose work overlaps on the GPU (other streams, other host threads) race on
 * it: order them on one stream, or synchronise between them. */
ks_status ks_chain_noalloc(const void *X, const void *const *factors,
                           const ks_pattern *patterns, int n_factors,
                           int64_t batch, void *Y, int dtype, void *stream);

/* Hierarchical butterfly factorization (the producer of butterfly chains):
 * fits the 2^log2n x 2^log2n dense matrix A (row-major, the K of Y = X K^T)
 * with the butterfly factors F_k = (2^(k-1), 2, 2, 2^(log2n-k)), k = 1..log2n,
 * F_1 applied first, so that ks_chain(X, factors, patterns) ~ X A^T.
 * The factor range is split in the middle recursively; each split fits two
 * chainable KS factors to the current KS product block by block with its best
 * rank-one approximation (power iteration from the block's largest-norm row,
 * a fixed number of steps).  A product of butterfly factors is recovered
 * exactly up to rounding; for other matrices the blocks' rank-one fits are
 * exact only as far as the power iteration has converged.  Each factor's
 * split sign makes the largest entry of its row part positive.
 * A and factors[0 .. log2n-1] are DEVICE fp32 arrays (factor k-1 holds
 * 2^(log2n+1) values [a][d][b][c]); dtype KS_F32 (KS_BF16: KS_ERR_UNSUPPORTED).
 * 1 <= log2n <= 14.  Intermediates come from the library's pool (stream-
 * ordered, freed before return). */
ks_status ks_butterfly_factorize(const void *A, int log2n, void *const *factors,
                                 int dtype, void *stream);

/* The library's workspace memory (not part of the paper's operation; for
 * callers that budget device memory).  *allocations (if non-NULL) receives
 * the number of workspace allocations the library has made from its pools
 * since the process started, on all devices; *reserved_bytes (if non-NULL)
 * the device memory the pool of the current device holds now (it keeps freed
 * workspace for later calls, see ks_chain).  Host-only apart from the pool
 * query; KS_ERR_CUDA if the current device has no pool. */
ks_status ks_workspace_info(int64_t *allocations, int64_t *reserved_bytes);

/* Measurement helper (not part of the paper's operation): the FP32 FMA
 * throughput of the current device's CUDA cores, the peak that bounds the
 * fp32 products.  Launches `blocks` blocks of 256 threads on `stream`; every
 * thread issues iters x 8 packed FMAs (fma.rn.f32x2, four flops each), so a
 * launch is blocks * 256 * iters * 32 flop.  out is a DEVICE array of
 * `blocks` floats (a checksum per block, so no work is optimised away).
 * Time it with events on `stream`.  KS_ERR_INVALID_ARG for a null out,
 * non-positive blocks, or iters not a positive multiple of 16. */
ks_status ks_fma_rate_probe(float *out, int blocks, int64_t iters, void *stream);

/* Fault injection for tests (read on every call, host side):
 *   KS_FAULT_INJECT=alloc    every workspace allocation fails: the entry
 *                            points that need one return KS_ERR_ALLOC before
 *                            launching anything (ks_matmul reads the values in
 *                            place instead);
 *   KS_FAULT_INJECT=timeout  the tensor-core kernels' pipeline waits (the
 *                            product's and the bf16 dV's) give up at once
 *                            instead of after about one second: the kernel
 *                            abandons its work (its output is unspecified),
 *                            drains its copies, frees its tensor memory and
 *                            returns, and the next ks_sync_status reports
 *                            KS_ERR_TIMEOUT.
 * Unset (or any other value), nothing is injected. */

/* Message for the last non-OK status returned on this host thread ("" if none). */
const char *ks_last_error(void);

/* Static name of a status code. */
const char *ks_status_string(int status);

/* Synchronises `stream`, then reports (and clears) the device-side status
 * word of the current device: KS_ERR_TIMEOUT if a bounded wait inside a
 * kernel gave up since the last call, KS_ERR_CUDA if the stream itself
 * failed, KS_OK otherwise. */
ks_status ks_sync_status(void *stream);

/* Library version, major*10000 + minor*100 + patch. */
int ks_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KS_B200_KS_H */
