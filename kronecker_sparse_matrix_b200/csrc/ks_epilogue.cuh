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

// GELU, tanh form: z (1 + tanh(u)) / 2 with u = sqrt(2/pi) (z + 0.044715 z^3),
// tanh(u) = 1 - 2 / (1 + e^(2u)) (exact identity; u clamped to [-15, 15], where
// tanh is +-1 to fp32 precision, so e^(2u) stays finite), e^x from the
// __expf intrinsic.  Its error is a few fp32 ulps of tanh, far inside the
// fp32 product tolerance.
__device__ __forceinline__ float gelu_tanh_f(float z) {
    float u = 0.7978845608028654f * (z + 0.044715f * z * z * z);
    u = fminf(fmaxf(u, -15.f), 15.f);
    const float t = 1.f - __fdividef(2.f, 1.f + __expf(2.f * u));
    return 0.5f * z * (1.f + t);
}

// GELU, tanh form, with the hardware tanh approximation (tanh.approx.f32,
// relative error about 2^-11): for the tensor-core outputs, whose tolerance
// (bf16 rounding, TF32 operands) is far coarser than that.
__device__ __forceinline__ float tanh_hw(float u) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(u));
    return t;
}
__device__ __forceinline__ float gelu_tanh_hw(float z) {
    const float u = 0.7978845608028654f * fmaf(0.044715f * z, z * z, z);
    return 0.5f * z * (1.f + tanh_hw(u));
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

// ep_act_array with the hardware tanh for the tanh form of GELU (tensor-core
// epilogues only).
template <int N>
__device__ __forceinline__ void ep_act_array_hw(float (&v)[N], int act) {
    if (act == 2) {
#pragma unroll
        for (int e = 0; e < N; ++e) v[e] = gelu_tanh_hw(v[e]);
    } else {
        ep_act_array(v, act);
    }
}

// acc + bias[col] (when bias is non-null), then the activation.
template <typename T>
__device__ __forceinline__ float ep_apply(float acc, const T *bias, long long col, int act) {
    if (bias) acc += ep_bias(bias, col);
    return act ? ep_act_fn(acc, act) : acc;
}

}  // namespace ks
