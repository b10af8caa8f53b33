// ks_chain_noalloc: a chain of KS factors that allocates no device memory.
//
// ks_chain keeps its two ping-pong intermediates in stream-ordered
// allocations.  Some callers must not allocate device memory once they are
// running: their device memory belongs to another allocator (a framework's
// caching pool that must account for every byte), or they run
// latency-critical loops where an allocation, and the synchronisation it may
// bring, is not allowed.  For them the intermediates live in one fixed array
// of this file, reserved on every device that loads the library and kept until
// the process exits.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "ks.h"
#include "ks_internal.h"

namespace {

// Two intermediates of at most kHalfBytes each.
constexpr size_t kScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr size_t kHalfBytes = kScratchBytes / 2;

static __device__ __align__(256) unsigned char g_chain_scratch[kScratchBytes];

// Device address of g_chain_scratch, looked up once per device with that
// device current (host code may not use the symbol itself as an address).
cudaError_t scratch_address(void **out) {
    static std::mutex mu;
    static void *addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_chain_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" ks_status ks_chain_noalloc(const void *X, const void *const *factors, const ks_pattern *patterns,
                                      int n_factors, int64_t batch, void *Y, int dtype, void *stream) {
    using ks::record_error;
    if (dtype != KS_F32 && dtype != KS_TF32 && dtype != KS_BF16)
        return record_error(KS_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (n_factors <= 0 || !factors || !patterns)
        return record_error(KS_ERR_INVALID_ARG, "need n_factors > 0 and non-null factors/patterns");
    if (batch < 0) return record_error(KS_ERR_INVALID_ARG, "batch must be >= 0 (got %lld)", (long long)batch);
    const int elem = dtype == KS_BF16 ? 2 : 4;
    int64_t widest = 0;
    for (int t = 0; t < n_factors; ++t) {
        const ks_pattern &q = patterns[t];
        if (q.a <= 0 || q.b <= 0 || q.c <= 0 || q.d <= 0)
            return record_error(KS_ERR_INVALID_ARG, "factor %d: pattern entries must be positive", t);
        if (q.a > INT32_MAX / q.b || q.a * q.b > INT32_MAX / q.d || q.a > INT32_MAX / q.c ||
            q.a * q.c > INT32_MAX / q.d)
            return record_error(KS_ERR_INVALID_ARG, "factor %d: width exceeds 2^31", t);
        if (t > 0) {
            const ks_pattern &r = patterns[t - 1];
            if (r.a * r.b * r.d != q.a * q.c * q.d)
                return record_error(KS_ERR_INVALID_ARG, "factor %d has input width %lld but factor %d outputs %lld", t,
                                    (long long)(q.a * q.c * q.d), t - 1, (long long)(r.a * r.b * r.d));
        }
        if (!factors[t]) return record_error(KS_ERR_INVALID_ARG, "factor %d is null", t);
        if (t < n_factors - 1) widest = std::max<int64_t>(widest, q.a * q.b * q.d);
    }
    if (batch == 0) return KS_OK;
    if (!X || !Y) return record_error(KS_ERR_INVALID_ARG, "X and Y must be non-null");
    // Every product runs with Problem::no_workspace: the fp32 kernel reads the
    // values in place instead of staging a transposed copy in a pooled workspace.
    if (n_factors == 1) {
        const ks_pattern &q = patterns[0];
        return ks::matmul_no_workspace(X, factors[0], q.a, q.b, q.c, q.d, batch, Y, dtype, stream);
    }
    if (widest > (int64_t)(kHalfBytes / elem) / batch)
        return record_error(KS_ERR_INVALID_ARG,
                            "an intermediate of %lld x %lld elements exceeds the fixed scratch: at most %zu bytes "
                            "per intermediate (batch x widest intermediate width x element size)",
                            (long long)batch, (long long)widest, kHalfBytes);
    void *scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess)
        return record_error(KS_ERR_CUDA, "looking up the chain scratch: %s", cudaGetErrorString(e));
    unsigned char *half[2] = {static_cast<unsigned char *>(scratch), static_cast<unsigned char *>(scratch) + kHalfBytes};
    const void *src = X;
    for (int t = 0; t < n_factors; ++t) {
        const ks_pattern &q = patterns[t];
        void *dst = (t == n_factors - 1) ? Y : static_cast<void *>(half[t & 1]);
        ks_status s = ks::matmul_no_workspace(src, factors[t], q.a, q.b, q.c, q.d, batch, dst, dtype, stream);
        if (s != KS_OK) return s;
        src = dst;
    }
    return KS_OK;
}
