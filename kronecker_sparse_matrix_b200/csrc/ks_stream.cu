// Streaming kernels for KS products whose blocks are tiny (b, c <= 8, e.g. the
// 2x2 blocks of a butterfly factor), and the catch-all path for any pattern
// and any element-aligned pointers.
//
// Y[n, i*b*d + k*d + l] = sum_j values[i, l, k, j] * X[n, i*c*d + j*d + l]
// (KS factor I_a (x) 1_{b x c} (x) I_d; taxoreview.com page on Kronecker-sparse
// matrix multiplication, first abstract: butterfly matrices are products of
// such factors).
//
// With b and c this small there is no reuse worth staging: every output reads
// its c inputs straight from HBM (through L1) and the kernel is bound by HBM
// bandwidth (2 flop per 4..8 bytes moved).  The vector kernel gives each
// thread one (row n, block i, group of VEC consecutive l) and all b outputs of
// it, so X is read once with 16-byte loads and Y is written with 16-byte
// stores, both coalesced across the warp (consecutive threads take
// consecutive l groups).  The scalar kernel (any d, any alignment) gives each
// thread one output element.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "ks_internal.h"

namespace ks {
namespace {

template <typename T> struct Vec16;  // 16 bytes of T
template <> struct Vec16<float> {
    static constexpr int N = 4;
    __device__ static void load(const float *p, float (&v)[4]) {
        float4 t = __ldg(reinterpret_cast<const float4 *>(p));
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    }
    __device__ static void store(float *p, const float (&v)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const __nv_bfloat16 *p, float (&v)[8]) {
        uint4 t = __ldg(reinterpret_cast<const uint4 *>(p));
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&t);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float2 f = __bfloat1622float2(h[q]);
            v[2 * q] = f.x;
            v[2 * q + 1] = f.y;
        }
    }
    __device__ static void store(__nv_bfloat16 *p, const float (&v)[8]) {
        uint4 t;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&t);
#pragma unroll
        for (int q = 0; q < 4; ++q) h[q] = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
        *reinterpret_cast<uint4 *>(p) = t;
    }
};

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void from_f(float &o, float v) { o = v; }
__device__ __forceinline__ void from_f(__nv_bfloat16 &o, float v) { o = __float2bfloat16_rn(v); }

// One thread per (n, i, l-group of VEC); loops over k in chunks of KB.
// Requires d % VEC == 0 and 16-byte aligned X, Y (then every row offset is
// 16-byte aligned too, since a*c*d and a*b*d are multiples of VEC).
template <typename T, int KB>
__global__ void __launch_bounds__(256) stream_vec_kernel(const T *__restrict__ X, const T *__restrict__ V,
                                                         T *__restrict__ Y, long long total, int a, int b,
                                                         int c, int d) {
    constexpr int VEC = Vec16<T>::N;
    const int dq = d / VEC;
    const long long in_f = (long long)a * c * d, out_f = (long long)a * b * d;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += stride) {
        const int lq = (int)(t % dq);
        const long long ni = t / dq;
        const int i = (int)(ni % a);
        const long long n = ni / a;
        const int l0 = lq * VEC;
        const T *x = X + n * in_f + (long long)i * c * d + l0;
        T *y = Y + n * out_f + (long long)i * b * d + l0;
        // values[i][l0 + e][k][j] = v[(e * b + k) * c + j]
        const T *v = V + ((long long)i * d + l0) * b * c;
        for (int k0 = 0; k0 < b; k0 += KB) {
            float acc[KB][VEC];
#pragma unroll
            for (int kk = 0; kk < KB; ++kk)
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[kk][e] = 0.f;
            for (int j = 0; j < c; ++j) {
                float xv[VEC];
                Vec16<T>::load(x + (long long)j * d, xv);
#pragma unroll
                for (int kk = 0; kk < KB; ++kk) {
                    const int k = k0 + kk;
                    if (k < b) {
#pragma unroll
                        for (int e = 0; e < VEC; ++e)
                            acc[kk][e] = fmaf(to_f(__ldg(v + ((long long)e * b + k) * c + j)), xv[e], acc[kk][e]);
                    }
                }
            }
#pragma unroll
            for (int kk = 0; kk < KB; ++kk) {
                const int k = k0 + kk;
                if (k < b) Vec16<T>::store(y + (long long)k * d, acc[kk]);
            }
        }
    }
}

// One thread per output element; any pattern, element-aligned pointers.
template <typename T>
__global__ void __launch_bounds__(256) stream_scalar_kernel(const T *__restrict__ X, const T *__restrict__ V,
                                                            T *__restrict__ Y, long long total, int a, int b,
                                                            int c, int d) {
    const long long in_f = (long long)a * c * d, out_f = (long long)a * b * d;
    const long long bd = (long long)b * d;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += stride) {
        const long long n = t / out_f;
        const long long r = t - n * out_f;
        const int i = (int)(r / bd);
        const long long rem = r - (long long)i * bd;
        const int k = (int)(rem / d);
        const int l = (int)(rem - (long long)k * d);
        const T *x = X + n * in_f + (long long)i * c * d + l;
        const T *v = V + (((long long)i * d + l) * b + k) * c;
        float acc = 0.f;
        for (int j = 0; j < c; ++j) acc = fmaf(to_f(__ldg(v + j)), to_f(__ldg(x + (long long)j * d)), acc);
        from_f(Y[t], acc);
    }
}

int grid_for(long long work, int threads) {
    long long blocks = (work + threads - 1) / threads;
    long long cap = (long long)sm_count() * 16;
    return (int)std::max<long long>(1, std::min(blocks, cap));
}

template <typename T>
cudaError_t launch_typed(const Problem &p) {
    constexpr int VEC = Vec16<T>::N;
    const T *X = static_cast<const T *>(p.X);
    const T *V = static_cast<const T *>(p.V);
    T *Y = static_cast<T *>(p.Y);
    const bool aligned = (reinterpret_cast<uintptr_t>(p.X) % 16 == 0) && (reinterpret_cast<uintptr_t>(p.Y) % 16 == 0);
    if (aligned && p.d % VEC == 0) {
        const long long total = p.batch * p.a * (p.d / VEC);
        if (p.b <= 2)
            stream_vec_kernel<T, 2><<<grid_for(total, 256), 256, 0, p.stream>>>(X, V, Y, total, (int)p.a, (int)p.b,
                                                                               (int)p.c, (int)p.d);
        else
            stream_vec_kernel<T, 4><<<grid_for(total, 256), 256, 0, p.stream>>>(X, V, Y, total, (int)p.a, (int)p.b,
                                                                               (int)p.c, (int)p.d);
    } else {
        const long long total = p.batch * p.out_features();
        stream_scalar_kernel<T><<<grid_for(total, 256), 256, 0, p.stream>>>(X, V, Y, total, (int)p.a, (int)p.b,
                                                                            (int)p.c, (int)p.d);
    }
    return cudaGetLastError();
}

}  // namespace

bool stream_supported(const Problem &) { return true; }

cudaError_t launch_stream(const Problem &p) {
    if (p.dtype == KS_BF16) return launch_typed<__nv_bfloat16>(p);
    return launch_typed<float>(p);  // KS_F32, and KS_TF32 computed in full fp32
}

}  // namespace ks
