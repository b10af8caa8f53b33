// Fused epilogue of a KS product, applied to each fp32 accumulator before it
// is stored: y = act(acc + bias[column]) (the MLP shapes' bias and
// activation).  act: 0 none, 1 ReLU, 2 GELU in its tanh form, 3 GELU in its
// erf form z * Phi(z).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace ks {

__device__ __forceinline__ float ep_bias(const float *b, long long col) { return __ldg(b + col); }
__device__ __forceinline__ float ep_bias(const __nv_bfloat16 *b, long long col) {
    return __bfloat162float(b[col]);
}

// GELU, tanh form: z (1 + tanh(u)) / 2 with u = sqrt(2/pi) (z + 0.044715 z^3).
// Since (1 + tanh(u)) / 2 = 1 / (1 + e^(-2u)) (the logistic function of 2u)
// and e^x = 2^(x log2 e), the value is z / (1 + 2^s) with
//     s = -2 log2(e) u = z (A + B z^2),  A = -2 log2(e) sqrt(2/pi),  B = 0.044715 A,
// evaluated with the PTX instructions ex2.approx and rcp.approx (each about
// 2^-22 relative error): three multiplies, one FMA and one add in the FP32
// pipe.  Large |z| needs no clamp: for z very negative s overflows to +inf,
// 2^s = inf and the reciprocal is 0 (output -0); for z very positive 2^s = 0
// and the output is z.  The error is a few fp32 ulps, far inside the fp32
// product tolerance.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kGeluA = -2.0f * 1.4426950408889634f * 0.7978845608028654f;
constexpr float kGeluB = 0.044715f * kGeluA;
__device__ __forceinline__ float gelu_tanh_f(float z) {
    const float s = z * fmaf(z * z, kGeluB, kGeluA);
    return z * rcp_approx(1.f + ex2_approx(s));
}
// The same on two values with the packed fp32 instructions of sm_100
// (add/mul/fma.rn.f32x2): 2.5 FP32-pipe instructions per output.
__device__ __forceinline__ float2 gelu_tanh_f2(float2 z) {
    const float2 q = __ffma2_rn(__fmul2_rn(z, z), make_float2(kGeluB, kGeluB), make_float2(kGeluA, kGeluA));
    const float2 s = __fmul2_rn(z, q);
    const float2 den = __fadd2_rn(make_float2(ex2_approx(s.x), ex2_approx(s.y)), make_float2(1.f, 1.f));
    return __fmul2_rn(z, make_float2(rcp_approx(den.x), rcp_approx(den.y)));
}

// The hardware tanh approximation (tanh.approx.f32, relative error about
// 2^-11), for GELU on the tensor-core outputs, whose tolerance (bf16 rounding,
// TF32 operands) is far coarser than that.
__device__ __forceinline__ float tanh_hw(float u) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(u));
    return t;
}
// GELU, erf form: z Phi(z) = z (1 + erf(z / sqrt 2)) / 2, CUDA's erff.
__device__ __forceinline__ float gelu_erf_f(float z) { return 0.5f * z * (1.f + erff(z * 0.7071067811865476f)); }

__device__ __forceinline__ float ep_act_fn(float z, int act) {
    switch (act) {
        case 1: return fmaxf(z, 0.f);
        case 2: return gelu_tanh_f(z);
        case 3: return gelu_erf_f(z);
        default: return z;
    }
}

// The activation over a whole array, the choice made once outside the
// element loop so the N elements are independent chains the scheduler can
// interleave.
template <int N>
__device__ __forceinline__ void ep_act_array(float (&v)[N], int act) {
    switch (act) {
        case 1:
#pragma unroll
            for (int e = 0; e < N; ++e) v[e] = fmaxf(v[e], 0.f);
            break;
        case 2:
#pragma unroll
            for (int e = 0; e < N; ++e) v[e] = gelu_tanh_f(v[e]);
            break;
        case 3:
#pragma unroll
            for (int e = 0; e < N; ++e) v[e] = gelu_erf_f(v[e]);
            break;
        default: break;
    }
}

// acc + bias[col] (when bias is non-null), then the activation.
template <typename T>
__device__ __forceinline__ float ep_apply(float acc, const T *bias, long long col, int act) {
    if (bias) acc += ep_bias(bias, col);
    return act ? ep_act_fn(acc, act) : acc;
}

}  // namespace ks
