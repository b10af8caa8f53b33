// Fused butterfly chain: the twelve KS factors (2^(k-1), 2, 2, 2^(12-k)),
// k = 1..12 (factor 1 applied first), of a 4096 x 4096 butterfly matrix,
// applied to blocks of rows in one kernel.
//
// A butterfly matrix is a product of KS factors with 2 x 2 blocks
// (taxoreview.com page on Kronecker-sparse matrix multiplication, first
// abstract).  Factor k of width 4096 has d = 2^(12-k), so it mixes the pair
// of activation entries whose indices differ in bit p = 12 - k:
//     y[e | 0<<p] = V[q][0][0] x[e | 0<<p] + V[q][0][1] x[e | 1<<p]
//     y[e | 1<<p] = V[q][1][0] x[e | 0<<p] + V[q][1][1] x[e | 1<<p]
// with values[i][l][k][j] at q = i*d + l, i.e. q = e with bit p removed.
//
// Applied one factor at a time, a chain moves the whole activation through
// HBM twelve times.  Here a CTA holds R rows and runs the twelve factors as
// three radix-16 passes over the index digits (bits 11-8, 7-4, 3-0): in each
// pass a thread owns the 16 entries that differ in that digit, for R rows, in
// registers, and applies four factors there.  Between passes the rows go
// through shared memory in an XOR-swizzled order in which all three thread
// mappings are free of bank conflicts.  X is read once and Y written once.
//
// Weights.  In passes 1 and 2 a warp's lanes take consecutive pairs, so each
// weight load is coalesced; they come from L2 (where the 12 x 2048 pairs stay)
// once per R rows.  In pass 3 the eight pairs of a thread are one contiguous
// line and a warp's load would touch 32 lines, so factors 9-12 are copied once
// per CTA into shared memory as fp32, line t (the thread's) with its eight
// 16-byte slots rotated by t & 7: both the coalesced copy and the per-thread
// reads are then free of bank conflicts.  (Keeping bf16 weights as bf16 there,
// with 8 rows per block, measured slower.)
//
// Rounding: fp32 FMAs, y = fma(V[k][1], x1, V[k][0] * x0), intermediates kept
// in fp32 (bf16 chains round only the final output).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "ks_internal.h"

namespace ks {
namespace {

constexpr int kWidth = 4096;
constexpr int kThreads = 256;

template <typename T> struct BflyIO;
template <> struct BflyIO<float> {
    __device__ static float load(const float *p) { return __ldg(p); }
    __device__ static float4 weights(const float *v, int q) { return __ldg(reinterpret_cast<const float4 *>(v) + q); }
    __device__ static void store16(float *p, const float (&v)[16]) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
            reinterpret_cast<float4 *>(p)[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
    }
};
template <> struct BflyIO<__nv_bfloat16> {
    __device__ static float load(const __nv_bfloat16 *p) { return __bfloat162float(p[0]); }
    __device__ static float4 weights(const __nv_bfloat16 *v, int q) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(v) + q);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        return make_float4(lo.x, lo.y, hi.x, hi.y);
    }
    __device__ static void store16(__nv_bfloat16 *p, const float (&v)[16]) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            uint4 o;
            __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
            for (int q = 0; q < 4; ++q) h[q] = __floats2bfloat162_rn(v[8 * u + 2 * q], v[8 * u + 2 * q + 1]);
            reinterpret_cast<uint4 *>(p)[u] = o;
        }
    }
};

struct BflyParams {
    const void *X;
    void *Y;
    long long N;
    const void *V[12];  // factor k + 1 at V[k]
};

// One factor on a thread's digit: the 16 entries v[r][m] of row r have indices
// e(m) = base | m << SHIFT, and the factor mixes bit p = SHIFT + S, i.e. digit
// bit S.  The weight index of the pair (m, m | 1<<S) is e(m) with bit p
// removed, which is qbase + qoff(m) with qoff a compile-time constant.
template <typename T, int R, int SHIFT, int S>
__device__ __forceinline__ void apply_factor(float (&v)[R][16], const T *V, int qbase) {
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        if (m & (1 << S)) continue;
        // e(m) = base | m << SHIFT; removing bit SHIFT + S keeps the digit's
        // bits below S in place and moves the ones above S down by one.
        constexpr int lowmask = (1 << S) - 1;
        const int qoff = ((m >> (S + 1)) << (SHIFT + S)) | ((m & lowmask) << SHIFT);
        const float4 w = BflyIO<T>::weights(V, qbase + qoff);
        const int m1 = m | (1 << S);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float x0 = v[r][m], x1 = v[r][m1];
            v[r][m] = fmaf(w.y, x1, w.x * x0);
            v[r][m1] = fmaf(w.w, x1, w.z * x0);
        }
    }
}

// Pass-3 factor from the resident copy: the k-th pair of thread t at slot
// k ^ tx of line t (tx = t & 7).
template <int R, int S>
__device__ __forceinline__ void apply_factor_res(float (&v)[R][16], const float4 *line, int tx) {
    int k = 0;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        if (m & (1 << S)) continue;
        const float4 w = line[k ^ tx];
        ++k;
        const int m1 = m | (1 << S);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float x0 = v[r][m], x1 = v[r][m1];
            v[r][m] = fmaf(w.y, x1, w.x * x0);
            v[r][m1] = fmaf(w.w, x1, w.z * x0);
        }
    }
}
// Shared-memory position of entry e = (A, B, C) digits (bits 11-8, 7-4, 3-0):
//   A*256 + ((B ^ A) & 15) * 16 + (C ^ ((B >> 1) | (A & 1) << 3)),
// a bijection on 0..4095 under which, for every pass's thread mapping, the 32
// lanes of a warp touch 32 distinct banks.
__device__ __forceinline__ int swz(int e) {
    const int A = e >> 8, B = (e >> 4) & 15, C = e & 15;
    return (A << 8) | (((B ^ A) & 15) << 4) | (C ^ ((B >> 1) | ((A & 1) << 3)));
}

template <typename T, int R>
__global__ void __launch_bounds__(kThreads, 1) butterfly12_kernel(const BflyParams p) {
    // R rows of 4096 fp32 in swizzled order, then factors 9-12's weights
    extern __shared__ float sm[];
    const T *X = static_cast<const T *>(p.X);
    T *Y = static_cast<T *>(p.Y);
    const int t = threadIdx.x;
    // Pass 1: thread t = (B, C), digit A varies: e = A << 8 | t.
    //   swz = A << 8 | (u1 ^ (A << 4 | (A & 1) << 3)), u1 = swz(t).
    // Pass 2: thread t = (A, C) = (t >> 4, t & 15), digit B varies.
    //   swz = u2 ^ (B << 4 | B >> 1), u2 = swz(A << 8 | C).
    // Pass 3: thread t = (A, B), digit C varies: e = t << 4 | C.
    //   swz = u3 ^ C, u3 = swz(t << 4).
    const int u1 = swz(t);
    const int base2 = ((t >> 4) << 8) | (t & 15);
    const int u2 = swz(base2);
    const int u3 = swz(t << 4);
    // Weight index bases (q without the digit's contribution).
    const int q1 = t;                                 // pass 1: bits 7-0 stay below p
    const int q2 = ((t >> 4) << 7) | (t & 15);        // pass 2: A moves down one bit
    const T *V[12];
#pragma unroll
    for (int k = 0; k < 12; ++k) V[k] = static_cast<const T *>(p.V[k]);

    // factors 9-12 into shared memory: pair g of factor f (g = t + 256 i, read
    // coalesced) goes to line g >> 3, slot (g & 7) ^ (line & 7); a thread's
    // reads in pass 3 are then conflict-free (lines are its own, slots rotate)
    float4 *res = reinterpret_cast<float4 *>(sm + R * kWidth);
#pragma unroll
    for (int f = 0; f < 4; ++f)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int g = t + 256 * i, line = g >> 3;
            res[f * 2048 + line * 8 + ((g & 7) ^ (line & 7))] = BflyIO<T>::weights(V[8 + f], g);
        }
    // (the first pass-1 -> pass-2 barrier orders these stores before any read)
    const float4 *res_t = res + t * 8;
    const int tx = t & 7;
    const long long n_blocks = (p.N + R - 1) / R;
    for (long long blk = blockIdx.x; blk < n_blocks; blk += gridDim.x) {
        const long long n0 = blk * R;
        float v[R][16];
        // ---- pass 1: factors 1-4 (bits 11, 10, 9, 8), straight from X
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const bool in = n0 + r < p.N;
            const T *x = X + (n0 + r) * kWidth + t;
#pragma unroll
            for (int A = 0; A < 16; ++A) v[r][A] = in ? BflyIO<T>::load(x + (A << 8)) : 0.f;
        }
        apply_factor<T, R, 8, 3>(v, V[0], q1);
        apply_factor<T, R, 8, 2>(v, V[1], q1);
        apply_factor<T, R, 8, 1>(v, V[2], q1);
        apply_factor<T, R, 8, 0>(v, V[3], q1);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int A = 0; A < 16; ++A)
                sm[r * kWidth + ((A << 8) | (u1 ^ ((A << 4) | ((A & 1) << 3))))] = v[r][A];
        __syncthreads();
        // ---- pass 2: factors 5-8 (bits 7, 6, 5, 4)
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int B = 0; B < 16; ++B) v[r][B] = sm[r * kWidth + (u2 ^ ((B << 4) | (B >> 1)))];
        apply_factor<T, R, 4, 3>(v, V[4], q2);
        apply_factor<T, R, 4, 2>(v, V[5], q2);
        apply_factor<T, R, 4, 1>(v, V[6], q2);
        apply_factor<T, R, 4, 0>(v, V[7], q2);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int B = 0; B < 16; ++B) sm[r * kWidth + (u2 ^ ((B << 4) | (B >> 1)))] = v[r][B];
        __syncthreads();
        // ---- pass 3: factors 9-12 (bits 3, 2, 1, 0), straight to Y
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int C = 0; C < 16; ++C) v[r][C] = sm[r * kWidth + (u3 ^ C)];
        apply_factor_res<R, 3>(v, res_t, tx);
        apply_factor_res<R, 2>(v, res_t + 2048, tx);
        apply_factor_res<R, 1>(v, res_t + 4096, tx);
        apply_factor_res<R, 0>(v, res_t + 6144, tx);
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (n0 + r < p.N) BflyIO<T>::store16(Y + (n0 + r) * kWidth + (t << 4), v[r]);
        __syncthreads();  // the next block's pass 1 overwrites shared memory
    }
}

template <typename T, int R>
cudaError_t launch_bfly(const BflyParams &p, cudaStream_t stream) {
    const size_t smem = (size_t)R * kWidth * sizeof(float) + 4 * 2048 * sizeof(float4);
    auto kern = butterfly12_kernel<T, R>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long n_blocks = (p.N + R - 1) / R;
    const long long grid = std::min<long long>(n_blocks, (long long)sm_count());
    kern<<<(int)grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool butterfly12_matches(const ks_pattern *patterns, int n) {
    if (n != 12) return false;
    for (int t = 0; t < 12; ++t) {
        const ks_pattern &q = patterns[t];
        if (q.a != (1LL << t) || q.b != 2 || q.c != 2 || q.d != (1LL << (11 - t))) return false;
    }
    return true;
}

bool butterfly12_supported(const void *X, const void *const *factors, void *Y, int dtype) {
    const uintptr_t align = dtype == KS_BF16 ? 8 : 16;
    if (reinterpret_cast<uintptr_t>(Y) % 16) return false;
    if (reinterpret_cast<uintptr_t>(X) % (dtype == KS_BF16 ? 2 : 4)) return false;
    for (int t = 0; t < 12; ++t)
        if (reinterpret_cast<uintptr_t>(factors[t]) % align) return false;
    return true;
}

cudaError_t launch_butterfly12(const void *X, const void *const *factors, long long batch, void *Y, int dtype,
                               cudaStream_t stream) {
    BflyParams p;
    p.X = X;
    p.Y = Y;
    p.N = batch;
    for (int t = 0; t < 12; ++t) p.V[t] = factors[t];
    // 6 rows per block: their 96 KB and the 128 KB of fp32 pass-3 weights fill
    // the 227 KB of shared memory a CTA may take
    if (dtype == KS_BF16) return launch_bfly<__nv_bfloat16, 6>(p, stream);
    return launch_bfly<float, 6>(p, stream);
}

}  // namespace ks
