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
#include <climits>
#include <cstdint>

#include "ks_epilogue.cuh"
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
                                                         int c, int d, const T *__restrict__ bias, int act) {
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
                if (k < b) {
                    if (bias) {
                        const long long col = (long long)i * b * d + (long long)k * d + l0;
#pragma unroll
                        for (int e = 0; e < VEC; ++e) acc[kk][e] += ep_bias(bias, col + e);
                    }
                    if (act) ep_act_array(acc[kk], act);
                    Vec16<T>::store(y + (long long)k * d, acc[kk]);
                }
            }
        }
    }
}

// One thread per output element; any pattern, element-aligned pointers.
template <typename T>
__global__ void __launch_bounds__(256) stream_scalar_kernel(const T *__restrict__ X, const T *__restrict__ V,
                                                            T *__restrict__ Y, long long total, int a, int b,
                                                            int c, int d, const T *__restrict__ bias, int act) {
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
        if (bias || act) acc = ep_apply(acc, bias, r, act);  // r = column of this output
        from_f(Y[t], acc);
    }
}

// Blocks per unit of the merged layout: the least U with U*C*D and U*B*D
// multiples of VEC (16-byte runs), or 0 if there is none up to VEC.
__host__ __device__ constexpr int merged_units(int B, int C, int D, int VEC) {
    for (int u = 1; u <= VEC; ++u)
        if ((u * C * D) % VEC == 0 && (u * B * D) % VEC == 0) return u;
    return 0;
}

// Register-weight streaming kernel for blocks of at most 4 x 4.  A thread owns
// one "unit" of a row and keeps the unit's weights in registers while it walks
// down a range of rows, so per row it moves only X in and Y out, as 16-byte
// loads and stores:
//   D == 0 (l-vector layout, d % VEC == 0): unit = (block i, VEC consecutive l);
//          input j is the VEC-run at i*C*d + j*d + l0, output k the run at
//          i*B*d + k*d + l0; weights values[i][l0 .. l0+VEC)[.][.] (contiguous);
//   D == d (merged layout, d small): unit = U consecutive blocks, whose U*C*d
//          inputs and U*B*d outputs are each one contiguous run; weights
//          values[i0 .. i0+U)[.][.][.] (contiguous).
// Threads form a TU x TR grid per CTA: TU consecutive units by TR row lanes.
// EP: fused epilogue (bias and activation) compiled in; the plain
// instantiation carries none of its code.
template <typename T, int B, int C, int D, bool EP>
__global__ void __launch_bounds__(256) stream_reg_kernel(const T *__restrict__ X, const T *__restrict__ V,
                                                         T *__restrict__ Y, long long N, int d, int units,
                                                         int in_f, int out_f, int tu_log2, int rows_per_cta,
                                                         const T *__restrict__ bias, int act) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int U = D == 0 ? 1 : merged_units(B, C, D, VEC);
    static_assert(U > 0, "no 16-byte merged layout for this block shape");
    constexpr int NL = D == 0 ? VEC : U * D;  // (block, l) lanes per unit
    constexpr int NW = NL * B * C;            // weights per unit
    const int tu = threadIdx.x & ((1 << tu_log2) - 1);
    const int tr = threadIdx.x >> tu_log2;
    const int TR = blockDim.x >> tu_log2;
    const int u = (blockIdx.x << tu_log2) + tu;
    if (u >= units) return;
    const long long n_begin = (long long)blockIdx.y * rows_per_cta + tr;
    const long long n_end = min(N, (long long)(blockIdx.y + 1) * rows_per_cta);

    int x_off, y_off, w_off;
    if constexpr (D == 0) {
        const int dq = d / VEC;
        const int i = u / dq, l0 = (u - i * dq) * VEC;
        x_off = i * C * d + l0;
        y_off = i * B * d + l0;
        w_off = (i * d + l0) * B * C;
    } else {
        x_off = u * (U * C * D);
        y_off = u * (U * B * D);
        w_off = u * NW;
    }
    // w[q] = values at w_off + q: lane e, output k, input j at q = (e*B + k)*C + j
    float w[NW];
#pragma unroll
    for (int q = 0; q < NW; q += VEC) {
        float t[VEC];
        Vec16<T>::load(V + w_off + q, t);
#pragma unroll
        for (int e = 0; e < VEC; ++e) w[q + e] = t[e];
    }

#pragma unroll 2
    for (long long n = n_begin; n < n_end; n += TR) {
        const T *x = X + n * in_f + x_off;
        T *y = Y + n * out_f + y_off;
        float xv[NL * C];  // xv[e*C + j]: lane e, input j
        if constexpr (D == 0) {
#pragma unroll
            for (int j = 0; j < C; ++j) {
                float t[VEC];
                Vec16<T>::load(x + j * d, t);
#pragma unroll
                for (int e = 0; e < VEC; ++e) xv[e * C + j] = t[e];
            }
        } else {
            // run layout [ub][j][l]; lane e = ub*D + l
#pragma unroll
            for (int q = 0; q < U * C * D; q += VEC) {
                float t[VEC];
                Vec16<T>::load(x + q, t);
#pragma unroll
                for (int r = 0; r < VEC; ++r) {
                    const int f = q + r, ub = f / (C * D), j = (f / D) % C, l = f % D;
                    xv[(ub * D + l) * C + j] = t[r];
                }
            }
        }
        float yv[NL * B];  // yv[e*B + k]
#pragma unroll
        for (int e = 0; e < NL; ++e)
#pragma unroll
            for (int k = 0; k < B; ++k) {
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < C; ++j) acc = fmaf(w[(e * B + k) * C + j], xv[e * C + j], acc);
                yv[e * B + k] = acc;
            }
        if (EP) {  // fused epilogue; column of (lane e, output k)
            if (bias) {
#pragma unroll
                for (int e = 0; e < NL; ++e)
#pragma unroll
                    for (int k = 0; k < B; ++k) {
                        const int col = D == 0 ? y_off + k * d + e : y_off + (e / D) * (B * D) + k * D + (e % D);
                        yv[e * B + k] += ep_bias(bias, col);
                    }
            }
            ep_act_array(yv, act);
        }
        if constexpr (D == 0) {
#pragma unroll
            for (int k = 0; k < B; ++k) {
                float t[VEC];
#pragma unroll
                for (int e = 0; e < VEC; ++e) t[e] = yv[e * B + k];
                Vec16<T>::store(y + k * d, t);
            }
        } else {
#pragma unroll
            for (int q = 0; q < U * B * D; q += VEC) {
                float t[VEC];
#pragma unroll
                for (int r = 0; r < VEC; ++r) {
                    const int f = q + r, ub = f / (B * D), k = (f / D) % B, l = f % D;
                    t[r] = yv[(ub * D + l) * B + k];
                }
                Vec16<T>::store(y + q, t);
            }
        }
    }
}

int grid_for(long long work, int threads) {
    long long blocks = (work + threads - 1) / threads;
    long long cap = (long long)sm_count() * 16;
    return (int)std::max<long long>(1, std::min(blocks, cap));
}

template <typename T, int B, int C, int D>
cudaError_t launch_reg(const Problem &p) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int U = D == 0 ? 1 : merged_units(B, C, D, VEC);
    const long long units = D == 0 ? p.a * p.d / VEC : p.a / U;
    int tu_log2 = 0;
    while ((1LL << tu_log2) < units && tu_log2 < 8) ++tu_log2;
    const int TU = 1 << tu_log2, TR = 256 / TU;
    const long long bx = (units + TU - 1) / TU;
    const long long target = (long long)sm_count() * 8;  // 8 CTAs of 256 threads per SM
    const long long max_by = std::min<long long>(65535, (p.batch + TR - 1) / TR);
    const long long by = std::max<long long>(1, std::min(max_by, (target + bx - 1) / bx));
    const long long rows_per_cta = (p.batch + by - 1) / by;
    if (bx > INT32_MAX || rows_per_cta > INT32_MAX) return cudaErrorInvalidConfiguration;
    auto kern = (p.bias || p.act) ? stream_reg_kernel<T, B, C, D, true> : stream_reg_kernel<T, B, C, D, false>;
    kern<<<dim3((unsigned)bx, (unsigned)by), 256, 0, p.stream>>>(
        static_cast<const T *>(p.X), static_cast<const T *>(p.V), static_cast<T *>(p.Y), p.batch, (int)p.d,
        (int)units, (int)p.in_features(), (int)p.out_features(), tu_log2, (int)rows_per_cta,
        static_cast<const T *>(p.bias), p.act);
    return cudaGetLastError();
}

// The register-weight kernel for (b, c) in {1, 2, 4}^2, if the layout allows:
// 16-byte aligned X, values and Y; d % VEC == 0 (l-vector layout), or d < VEC
// with a merged unit of U blocks dividing a.  cudaErrorNotSupported otherwise.
template <typename T, int B, int C>
cudaError_t launch_reg_bc(const Problem &p) {
    constexpr int VEC = Vec16<T>::N;
    if (p.d % VEC == 0) return launch_reg<T, B, C, 0>(p);
    switch (p.d) {
        case 1:
            if (merged_units(B, C, 1, VEC) && p.a % merged_units(B, C, 1, VEC) == 0) return launch_reg<T, B, C, 1>(p);
            break;
        case 2:
            if (merged_units(B, C, 2, VEC) && p.a % merged_units(B, C, 2, VEC) == 0) return launch_reg<T, B, C, 2>(p);
            break;
        case 4:
            if constexpr (VEC == 8) {
                if (merged_units(B, C, 4, VEC) && p.a % merged_units(B, C, 4, VEC) == 0)
                    return launch_reg<T, B, C, 4>(p);
            }
            break;
        default: break;
    }
    return cudaErrorNotSupported;
}

template <typename T, int B>
cudaError_t launch_reg_b(const Problem &p) {
    switch (p.c) {
        case 1: return launch_reg_bc<T, B, 1>(p);
        case 2: return launch_reg_bc<T, B, 2>(p);
        case 4: return launch_reg_bc<T, B, 4>(p);
        default: return cudaErrorNotSupported;
    }
}

template <typename T>
cudaError_t launch_reg_any(const Problem &p) {
    const uintptr_t al = reinterpret_cast<uintptr_t>(p.X) | reinterpret_cast<uintptr_t>(p.V) |
                         reinterpret_cast<uintptr_t>(p.Y);
    if (al % 16) return cudaErrorNotSupported;
    switch (p.b) {
        case 1: return launch_reg_b<T, 1>(p);
        case 2: return launch_reg_b<T, 2>(p);
        case 4: return launch_reg_b<T, 4>(p);
        default: return cudaErrorNotSupported;
    }
}

template <typename T>
cudaError_t launch_typed(const Problem &p) {
    constexpr int VEC = Vec16<T>::N;
    const T *X = static_cast<const T *>(p.X);
    const T *V = static_cast<const T *>(p.V);
    T *Y = static_cast<T *>(p.Y);
    const T *B = static_cast<const T *>(p.bias);
    const cudaError_t er = launch_reg_any<T>(p);
    if (er != cudaErrorNotSupported) return er;
    const bool aligned = (reinterpret_cast<uintptr_t>(p.X) % 16 == 0) && (reinterpret_cast<uintptr_t>(p.Y) % 16 == 0);
    if (aligned && p.d % VEC == 0) {
        const long long total = p.batch * p.a * (p.d / VEC);
        if (p.b <= 2)
            stream_vec_kernel<T, 2><<<grid_for(total, 256), 256, 0, p.stream>>>(X, V, Y, total, (int)p.a, (int)p.b,
                                                                               (int)p.c, (int)p.d, B, p.act);
        else
            stream_vec_kernel<T, 4><<<grid_for(total, 256), 256, 0, p.stream>>>(X, V, Y, total, (int)p.a, (int)p.b,
                                                                               (int)p.c, (int)p.d, B, p.act);
    } else {
        const long long total = p.batch * p.out_features();
        stream_scalar_kernel<T><<<grid_for(total, 256), 256, 0, p.stream>>>(X, V, Y, total, (int)p.a, (int)p.b,
                                                                            (int)p.c, (int)p.d, B, p.act);
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
