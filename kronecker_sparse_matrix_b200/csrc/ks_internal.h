// Internal interfaces between the C ABI (ks_api.cu), the pattern heuristic
// (ks_plan.cu) and the kernel families (ks_stream.cu, ks_fma.cu, ks_tc.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ks.h"

namespace ks {

// One KS product, after validation: Y = X K^T with K of pattern (a,b,c,d).
struct Problem {
    const void *X;
    const void *V;  // values[a][d][b][c]
    void *Y;
    int64_t a, b, c, d, batch;
    int dtype;      // ks_dtype
    cudaStream_t stream;
    // Fused epilogue Y = act(X K^T + bias): bias holds out_features() elements
    // of the storage dtype (or is null), act is a ks_activation.
    const void *bias = nullptr;
    int act = 0;
    // Set for callers that must not allocate: every kernel then works in the
    // caller's buffers only (the fp32 kernel reads the values in place instead
    // of staging a transposed copy in a pooled workspace).
    bool no_workspace = false;

    int64_t in_features() const { return a * c * d; }
    int64_t out_features() const { return a * b * d; }
    int elem_bytes() const { return dtype == KS_BF16 ? 2 : 4; }
};

// Tile choice of the CUDA-core gather-GEMM (see ks_fma.cu).
struct FmaConfig {
    int dl;  // l values per CTA (1, 2, 4 or 8)
    int wm;  // warps along rows per l   (warp tile 64 rows)
    int wk;  // warps along k per l      (warp tile 4*tn k)
    int tn;  // k per thread (8, 12 or 16)
};

// Tile choice of the tcgen05 block-GEMM (see ks_tc.cu).
struct TcConfig {
    int dl;  // l values per CTA
    int bk;  // k values per CTA tile (MMA N)
    int ct;  // j values per pipeline stage
};

struct Plan {
    int variant;  // ks_variant, never AUTO
    FmaConfig fma;
    TcConfig tc;
};

// Heuristic (ks_plan.cu).  Returns false if `variant` (possibly forced) cannot
// run this problem; `why` then says so.
bool make_plan(const Problem &p, int variant, Plan *out, const char **why);

// Capability checks used by the heuristic.
bool stream_supported(const Problem &p);
bool fma_supported(const Problem &p, const char **why);
bool tc_supported(const Problem &p, const char **why);
FmaConfig fma_choose(const Problem &p);
TcConfig tc_choose(const Problem &p);

// Launchers: return cudaSuccess or the launch error.  Pure device work on
// p.stream; no allocation, no synchronisation.
cudaError_t launch_stream(const Problem &p);
cudaError_t launch_fma(const Problem &p, const FmaConfig &cfg);
cudaError_t launch_fma32(const Problem &p, const FmaConfig &cfg);  // fp32, cp.async ring (ks_fma32.cu)
cudaError_t launch_tc(const Problem &p, const TcConfig &cfg);

// Gradients (ks_backward.cu).  dV[i][l][k][j] = sum_n dY[n,(i,k,l)] X[n,(i,j,l)]
// is computed over `splits` row ranges into fp32 partials W[split][a][d][b][c],
// then reduced into dV (dtype of dY/X).
struct DvProblem {
    const void *dY, *X;
    void *dV;
    int64_t a, b, c, d, batch;
    int dtype;
    cudaStream_t stream;
};
int dv_dl(int64_t d);
void dv_split(const DvProblem &q, int *splits, long long *rows_per_split);
cudaError_t launch_dv(const DvProblem &q, float *W, int splits, long long rows_per_split);
// dV on the tensor cores (ks_dv_tc.cu): bf16, d % 8 == 0, c % 16 == 0, c <= 64,
// b >= 128, 16-byte-aligned buffers; row ranges are multiples of 16.
bool dv_tc_supported(const DvProblem &q);
void dv_tc_split(const DvProblem &q, int *splits, long long *rows_per_split);
cudaError_t launch_dv_tc(const DvProblem &q, float *W, int splits, long long rows_per_split);
// The driver's cuTensorMapEncodeTiled (ks_tc.cu), or null when unavailable.
void *tensor_map_encoder();
// Bound of the tensor-core pipelines' mbarrier waits in ns (ks_tc.cu): about
// one second, or 0 under KS_FAULT_INJECT=timeout.
unsigned long long pipeline_wait_bound_ns();
// Column sums db[col] = sum_n dY[n][col] (ks_backward.cu): fp32 partial sums
// over `splits` row ranges into W[split][width], then added in range order.
void colsum_split(long long batch, long long width, int *splits, long long *rows_per_split);
cudaError_t launch_colsum(const void *dY, void *db, long long batch, long long width, int dtype, float *W, int splits,
                          long long rows_per_split, cudaStream_t stream);
// vt[blk][j][k] = v[blk][k][j] for `blocks` blocks of b x c (KS values transposed per (i, l)).
cudaError_t launch_transpose_blocks(const void *v, void *vt, int64_t blocks, int64_t b, int64_t c, int dtype,
                                    cudaStream_t stream);
// Two-factor fit of a KS product (ks_factorize.cu): P of pattern
// (a1, b1*b2, c1*c2, d2) -> V1 (a1, b1, c1, c2*d2) and V2 (a1*b1, b2, c2, d2),
// one best rank-one block per (i1, k1, j2, l2).  cudaErrorInvalidValue when a
// block (b2 x (c1 + 1) floats) exceeds fit_max_block_elems().
int fit_max_block_elems();
cudaError_t launch_rank1_fit(const float *P, float *V1, float *V2, int64_t a1, int64_t b1, int64_t c1, int64_t b2,
                             int64_t c2, int64_t d2, cudaStream_t stream);

// The library's retaining workspace pool of the current device (ks_api.cu).
cudaMemPool_t chain_pool();
// Stream-ordered allocation from chain_pool(); every successful one is counted
// (ks_workspace_info).  Returns cudaErrorMemoryAllocation without a pool.
cudaError_t pool_alloc(void **ptr, size_t bytes, cudaStream_t stream);

// One validated KS product with Problem::no_workspace set (ks_api.cu; used by
// ks_chain_noalloc).
ks_status matmul_no_workspace(const void *X, const void *V, int64_t a, int64_t b, int64_t c, int64_t d,
                              int64_t batch, void *Y, int dtype, void *stream);

// Fused 4096-wide butterfly chain (ks_butterfly.cu): the twelve factors
// (2^t, 2, 2, 2^(11-t)), t = 0..11, in that order.
bool butterfly12_matches(const ks_pattern *patterns, int n);
bool butterfly12_supported(const void *X, const void *const *factors, void *Y, int dtype);
cudaError_t launch_butterfly12(const void *X, const void *const *factors, long long batch, void *Y, int dtype,
                               cudaStream_t stream);

// Device status word (ks_api.cu): kernels OR these bits in on failure.
enum DeviceStatusBits : unsigned {
    kDevTimeout = 1u,
};
unsigned *device_status_ptr();  // address of the status word on the current device

// Number of SMs of the current device (cached per device).
int sm_count();

// Records the message ks_last_error() returns on this host thread and passes
// the status through (for entry points defined outside ks_api.cu).
ks_status record_error(ks_status s, const char *fmt, ...);

}  // namespace ks
