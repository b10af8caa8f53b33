// FP32 FMA throughput probe: the CUDA-core peak that bounds the fp32 KS
// products, measured on the device they run on instead of derived from unit
// counts and a nominal clock.
//
// Every thread runs `iters` rounds of eight independent chains of packed
// FMAs (fma.rn.f32x2: two FMAs, four flops per instruction) on registers;
// eight warps per scheduler and eight chains per thread cover the FMA
// latency.  The rounds are unrolled sixteen at a time, so the loop's own
// counter, compare and branch (which take issue slots and, for the integer
// arithmetic, pipe cycles) are one instruction in 40: the FMA pipes are the
// limit.  Each block writes one checksum (thread 0's sum, and any thread whose
// sum hits a value the arithmetic cannot produce), so the compiler keeps
// every chain.
#include <cuda_runtime.h>

#include <cstdint>

#include "ks.h"
#include "ks_internal.h"

namespace ks {
namespace {

constexpr int kProbeThreads = 256;
constexpr int kChains = 8;
constexpr int kUnroll = 16;  // rounds per loop iteration; iters is a multiple of it

__global__ void __launch_bounds__(kProbeThreads) fma_probe_kernel(float *out, int loops) {
    float2 acc[kChains];
#pragma unroll
    for (int k = 0; k < kChains; ++k)
        acc[k] = make_float2(1e-3f * (float)(threadIdx.x + k), 2e-3f * (float)(blockIdx.x + k));
    // |m| < 1 keeps every chain bounded: x -> m x + c converges to c / (1 - m)
    const float2 m = make_float2(0.999f, 0.998f), c = make_float2(1e-4f, -1e-4f);
    for (int it = 0; it < loops; ++it) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
#pragma unroll
            for (int k = 0; k < kChains; ++k) acc[k] = __ffma2_rn(acc[k], m, c);
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kChains; ++k) s += acc[k].x + acc[k].y;
    if (threadIdx.x == 0 || s == 12345.678f) out[blockIdx.x] = s;
}

}  // namespace
}  // namespace ks

extern "C" ks_status ks_fma_rate_probe(float *out, int blocks, int64_t iters, void *stream) {
    if (!out || blocks <= 0 || iters <= 0 || iters % ks::kUnroll || iters / ks::kUnroll > INT32_MAX)
        return ks::record_error(KS_ERR_INVALID_ARG,
                                "need out non-null, blocks > 0 and iters a positive multiple of %d", ks::kUnroll);
    if (reinterpret_cast<uintptr_t>(out) % 4)
        return ks::record_error(KS_ERR_MISALIGNED, "out is not aligned to its 4-byte element");
    ks::fma_probe_kernel<<<blocks, ks::kProbeThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        out, (int)(iters / ks::kUnroll));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return ks::record_error(KS_ERR_CUDA, "probe launch: %s (%s)", cudaGetErrorName(e), cudaGetErrorString(e));
    return KS_OK;
}
