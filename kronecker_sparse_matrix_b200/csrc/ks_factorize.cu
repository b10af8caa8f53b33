// Hierarchical butterfly factorization on the GPU (taxoreview.com page, third
// abstract: a matrix is split recursively into two
// factors with butterfly supports, each split a two-factor fixed-support
// factorization with exact recovery).
//
// Two chainable KS factors, K1 = (a1, b1, c1, d1) applied first and
// K2 = (a1*b1, b2, c2, d2) with d1 = c2*d2, multiply to the KS pattern
// (a1, b1*b2, c1*c2, d2) entry by entry:
//     P[i1][l2][k1*b2 + k2][j1*c2 + j2] = V2[i1*b1 + k1][l2][k2][j2] * V1[i1][j2*d2 + l2][k1][j1],
// so each b2 x c1 block B[k2][j1] of P (fixed i1, k1, j2, l2) is one column
// of V2 times one row of V1, and the fit is the block's best rank-one
// approximation s u v^T, written as sqrt(s) u and sqrt(s) v.
//
// rank1_fit_kernel: one CTA per block.  The block goes to shared memory
// (rows padded by one word); v starts as the block's largest-norm row (for
// a block that is exactly rank one this is already the answer), then
// kPowerIters power iterations v <- B^T B v / |B^T B v|; u = B v / s with
// s = |B v|.  The sign makes the largest-magnitude entry of v positive (the
// first on ties).  Blocks whose top two singular values are close converge
// slowly; the exact-recovery case (a product of butterfly factors) does not
// depend on the iteration count.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdint>

#include "ks_internal.h"

namespace ks {
namespace {

constexpr int kFitThreads = 256;
constexpr int kPowerIters = 24;
constexpr int kMaxBlockElems = 128 * 129;  // b2 x (c1 + 1) floats of shared memory

struct FitParams {
    const float *P;  // product values [a1][d2][b1*b2][c1*c2]
    float *V1;       // [a1][c2*d2][b1][c1]
    float *V2;       // [a1*b1][d2][b2][c2]
    int a1, b1, c1, b2, c2, d2;
};

__device__ float block_sum(float v, float *red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    float t = 0.f;
    if (threadIdx.x < 32) {
        t = threadIdx.x < (int)(blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (threadIdx.x == 0) red[0] = t;
    }
    __syncthreads();
    return red[0];
}

__global__ void __launch_bounds__(kFitThreads) rank1_fit_kernel(const FitParams p) {
    extern __shared__ float fsm[];
    const int b2 = p.b2, c1 = p.c1, ld = c1 + 1;
    float *B = fsm;                 // b2 x ld
    float *v = B + b2 * ld;         // c1
    float *w = v + c1;              // b2 (B v, then u)
    float *tmp = w + b2;            // c1
    float *red = tmp + c1;          // 32 (reductions)
    __shared__ int best_row;

    // block (i1, k1, j2, l2), l2 fastest
    int t = blockIdx.x;
    const int l2 = t % p.d2; t /= p.d2;
    const int j2 = t % p.c2; t /= p.c2;
    const int k1 = t % p.b1;
    const int i1 = t / p.b1;
    const int B_ = p.b1 * b2, C_ = c1 * p.c2;
    const float *src = p.P + ((long long)(i1 * p.d2 + l2) * B_ + (long long)k1 * b2) * C_ + j2;
    for (int e = threadIdx.x; e < b2 * c1; e += blockDim.x) {
        const int k2 = e / c1, j1 = e % c1;
        B[k2 * ld + j1] = src[(long long)k2 * C_ + (long long)j1 * p.c2];
    }
    __syncthreads();

    // start: the row of largest norm (smallest index on ties)
    if (threadIdx.x < 32) {
        float bn = -1.f;
        int bi = 0;
        for (int r = threadIdx.x; r < b2; r += 32) {
            float s = 0.f;
            for (int j = 0; j < c1; ++j) s = fmaf(B[r * ld + j], B[r * ld + j], s);
            if (s > bn) { bn = s; bi = r; }
        }
        for (int o = 16; o > 0; o >>= 1) {
            const float on = __shfl_xor_sync(0xffffffffu, bn, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (on > bn || (on == bn && oi < bi)) { bn = on; bi = oi; }
        }
        if (threadIdx.x == 0) best_row = bi;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < c1; j += blockDim.x) v[j] = B[best_row * ld + j];
    __syncthreads();
    {
        float s = 0.f;
        for (int j = threadIdx.x; j < c1; j += blockDim.x) s = fmaf(v[j], v[j], s);
        const float nrm = sqrtf(block_sum(s, red));
        const float inv = nrm > 0.f ? 1.f / nrm : 0.f;
        for (int j = threadIdx.x; j < c1; j += blockDim.x) v[j] *= inv;
        __syncthreads();
    }
    for (int it = 0; it < kPowerIters; ++it) {
        for (int r = threadIdx.x; r < b2; r += blockDim.x) {  // w = B v
            float s = 0.f;
            for (int j = 0; j < c1; ++j) s = fmaf(B[r * ld + j], v[j], s);
            w[r] = s;
        }
        __syncthreads();
        float s2 = 0.f;
        for (int j = threadIdx.x; j < c1; j += blockDim.x) {  // tmp = B^T w
            float s = 0.f;
            for (int r = 0; r < b2; ++r) s = fmaf(B[r * ld + j], w[r], s);
            tmp[j] = s;
            s2 = fmaf(s, s, s2);
        }
        const float nrm = sqrtf(block_sum(s2, red));
        const float inv = nrm > 0.f ? 1.f / nrm : 0.f;
        for (int j = threadIdx.x; j < c1; j += blockDim.x) v[j] = tmp[j] * inv;
        __syncthreads();
    }
    // u = B v, s = |u|
    float s2 = 0.f;
    for (int r = threadIdx.x; r < b2; r += blockDim.x) {
        float s = 0.f;
        for (int j = 0; j < c1; ++j) s = fmaf(B[r * ld + j], v[j], s);
        w[r] = s;
        s2 = fmaf(s, s, s2);
    }
    const float sig = sqrtf(block_sum(s2, red));
    // sign: the largest |v| entry positive (first on ties)
    if (threadIdx.x < 32) {
        float bm = -1.f;
        int bi = 0;
        for (int j = threadIdx.x; j < c1; j += 32)
            if (fabsf(v[j]) > bm) { bm = fabsf(v[j]); bi = j; }
        for (int o = 16; o > 0; o >>= 1) {
            const float om = __shfl_xor_sync(0xffffffffu, bm, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (om > bm || (om == bm && oi < bi)) { bm = om; bi = oi; }
        }
        if (threadIdx.x == 0) best_row = bi;
    }
    __syncthreads();
    const float sgn = v[best_row] < 0.f ? -1.f : 1.f;
    const float rs = sqrtf(sig);
    const float ru = sig > 0.f ? sgn * rs / sig : 0.f;  // sqrt(s) u = sqrt(s) (B v) / s
    const int a2i = i1 * p.b1 + k1, d1 = p.c2 * p.d2;
    for (int k2 = threadIdx.x; k2 < b2; k2 += blockDim.x)
        p.V2[((long long)(a2i * p.d2 + l2) * b2 + k2) * p.c2 + j2] = ru * w[k2];
    for (int j1 = threadIdx.x; j1 < c1; j1 += blockDim.x)
        p.V1[((long long)(i1 * d1 + j2 * p.d2 + l2) * p.b1 + k1) * c1 + j1] = sgn * rs * v[j1];
}

}  // namespace

int fit_max_block_elems() { return kMaxBlockElems; }

cudaError_t launch_rank1_fit(const float *P, float *V1, float *V2, int64_t a1, int64_t b1, int64_t c1, int64_t b2,
                             int64_t c2, int64_t d2, cudaStream_t stream) {
    if (b2 * (c1 + 1) > kMaxBlockElems) return cudaErrorInvalidValue;
    FitParams p{P, V1, V2, (int)a1, (int)b1, (int)c1, (int)b2, (int)c2, (int)d2};
    const long long blocks = a1 * b1 * c2 * d2;
    if (blocks > INT32_MAX) return cudaErrorInvalidValue;
    const size_t smem = (size_t)(b2 * (c1 + 1) + 2 * c1 + b2 + 32) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(rank1_fit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    rank1_fit_kernel<<<(int)blocks, kFitThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace ks
