// FP32 FMA throughput probe: the CUDA-core peak that bounds the fp32 KS
// products, measured on the device they run on instead of derived from unit
// counts and a nominal clock.
//
// Every thread runs `iters` rounds of eight independent chains of packed
// FMAs (fma.rn.f32x2: two FMAs, four flops per instruction) on registers;
// eight warps per scheduler and eight chains per thread cover the FMA
// latency, so the FMA pipes are the only limit.  Each block writes one
// checksum (thread 0's sum, and any thread whose sum hits a value the
// arithmetic cannot produce), so the compiler keeps every chain.
#include <cuda_runtime.h>

#include <cstdint>

#include "ks.h"
#include "ks_internal.h"

namespace ks {
namespace {

constexpr int kProbeThreads = 256;
constexpr int kChains = 8;

__global__ void __launch_bounds__(kProbeThreads) fma_probe_kernel(float *out, long long iters) {
    float2 acc[kChains];
#pragma unroll
    for (int k = 0; k < kChains; ++k)
        acc[k] = make_float2(1e-3f * (float)(threadIdx.x + k), 2e-3f * (float)(blockIdx.x + k));
    // |m| < 1 keeps every chain bounded: x -> m x + c converges to c / (1 - m)
    const float2 m = make_float2(0.999f, 0.998f), c = make_float2(1e-4f, -1e-4f);
    for (long long it = 0; it < iters; ++it) {
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
    if (!out || blocks <= 0 || iters <= 0)
        return ks::record_error(KS_ERR_INVALID_ARG, "need out non-null, blocks > 0 and iters > 0");
    if (reinterpret_cast<uintptr_t>(out) % 4)
        return ks::record_error(KS_ERR_MISALIGNED, "out is not aligned to its 4-byte element");
    ks::fma_probe_kernel<<<blocks, ks::kProbeThreads, 0, static_cast<cudaStream_t>(stream)>>>(out, (long long)iters);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return ks::record_error(KS_ERR_CUDA, "probe launch: %s (%s)", cudaGetErrorName(e), cudaGetErrorString(e));
    return KS_OK;
}
