// C ABI of the KS library: argument validation, dispatch to a kernel family,
// the chain executor and error reporting.  Everything here runs on the host;
// the only device work is the kernels the launchers enqueue and the chain's
// stream-ordered workspace.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <climits>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>

#include "ks.h"
#include "ks_internal.h"

namespace ks {
namespace {

thread_local char g_msg[512] = "";

ks_status fail(ks_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return s;
}

ks_status ok() { return KS_OK; }

// a*b with overflow check on non-negative operands.
bool mul_ok(int64_t a, int64_t b, int64_t *out) {
    if (a != 0 && b > INT64_MAX / a) return false;
    *out = a * b;
    return true;
}

bool ranges_overlap(const void *p, int64_t pbytes, const void *q, int64_t qbytes) {
    if (!p || !q || pbytes <= 0 || qbytes <= 0) return false;
    auto a0 = reinterpret_cast<uintptr_t>(p), b0 = reinterpret_cast<uintptr_t>(q);
    return a0 < b0 + (uintptr_t)qbytes && b0 < a0 + (uintptr_t)pbytes;
}

// Validates one factor's sizes; fills the element counts.
ks_status check_sizes(int64_t a, int64_t b, int64_t c, int64_t d, int64_t batch,
                      int64_t *in_f, int64_t *out_f, int64_t *nvals) {
    if (a <= 0 || b <= 0 || c <= 0 || d <= 0)
        return fail(KS_ERR_INVALID_ARG, "pattern entries must be positive (a=%lld b=%lld c=%lld d=%lld)",
                    (long long)a, (long long)b, (long long)c, (long long)d);
    if (batch < 0) return fail(KS_ERR_INVALID_ARG, "batch must be >= 0 (got %lld)", (long long)batch);
    int64_t ac, acd, ab, abd, abc, abcd, t1, t2;
    if (!mul_ok(a, c, &ac) || !mul_ok(ac, d, &acd) || !mul_ok(a, b, &ab) || !mul_ok(ab, d, &abd) ||
        !mul_ok(ab, c, &abc) || !mul_ok(abc, d, &abcd) || !mul_ok(std::max<int64_t>(batch, 1), acd, &t1) ||
        !mul_ok(std::max<int64_t>(batch, 1), abd, &t2) || !mul_ok(t1, 4, &t1) || !mul_ok(t2, 4, &t2) ||
        !mul_ok(abcd, 4, &abcd))
        return fail(KS_ERR_INVALID_ARG, "sizes overflow int64");
    // the kernels index rows with 32-bit feature offsets
    if (acd > INT32_MAX || abd > INT32_MAX || abcd / 4 > INT32_MAX)
        return fail(KS_ERR_INVALID_ARG, "a row or the values array exceeds 2^31 elements");
    *in_f = acd;
    *out_f = abd;
    *nvals = abcd / 4;
    return KS_OK;
}

ks_status check_dtype(int dtype) {
    if (dtype != KS_F32 && dtype != KS_TF32 && dtype != KS_BF16)
        return fail(KS_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    return KS_OK;
}

ks_status check_align(const void *p, int elem, const char *name) {
    if (reinterpret_cast<uintptr_t>(p) % (uintptr_t)elem != 0)
        return fail(KS_ERR_MISALIGNED, "%s is not aligned to its %d-byte element", name, elem);
    return KS_OK;
}

ks_status cuda_fail(cudaError_t e, const char *what) {
    return fail(KS_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// Validates a single product and builds the Problem; *noop set for batch == 0.
ks_status make_problem(const void *X, const void *V, int64_t a, int64_t b, int64_t c, int64_t d,
                       int64_t batch, void *Y, int dtype, void *stream, Problem *p, bool *noop) {
    ks_status s = check_dtype(dtype);
    if (s != KS_OK) return s;
    int64_t in_f = 0, out_f = 0, nvals = 0;
    if ((s = check_sizes(a, b, c, d, batch, &in_f, &out_f, &nvals)) != KS_OK) return s;
    *noop = (batch == 0);
    if (*noop) return KS_OK;
    if (!X || !V || !Y) return fail(KS_ERR_INVALID_ARG, "X, values and Y must be non-null");
    const int elem = dtype == KS_BF16 ? 2 : 4;
    if ((s = check_align(X, elem, "X")) != KS_OK) return s;
    if ((s = check_align(V, elem, "values")) != KS_OK) return s;
    if ((s = check_align(Y, elem, "Y")) != KS_OK) return s;
    const int64_t ybytes = batch * out_f * elem;
    if (ranges_overlap(Y, ybytes, X, batch * in_f * elem))
        return fail(KS_ERR_INVALID_ARG, "Y overlaps X");
    if (ranges_overlap(Y, ybytes, V, nvals * elem))
        return fail(KS_ERR_INVALID_ARG, "Y overlaps values");
    *p = Problem{X, V, Y, a, b, c, d, batch, dtype, static_cast<cudaStream_t>(stream)};
    return KS_OK;
}

ks_status run(const Problem &p, int variant) {
    Plan plan;
    const char *why = "";
    if (!make_plan(p, variant, &plan, &why))
        return fail(KS_ERR_UNSUPPORTED, "variant %d cannot run pattern (%lld,%lld,%lld,%lld) dtype %d: %s",
                    variant, (long long)p.a, (long long)p.b, (long long)p.c, (long long)p.d, p.dtype, why);
    cudaError_t e = cudaSuccess;
    switch (plan.variant) {
        case KS_VARIANT_STREAM: e = launch_stream(p); break;
        case KS_VARIANT_FMA: e = launch_fma(p, plan.fma); break;
        case KS_VARIANT_TC: e = launch_tc(p, plan.tc); break;
        default: return fail(KS_ERR_UNSUPPORTED, "no kernel for variant %d", plan.variant);
    }
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return ok();
}

// Device status word, one per device (a __device__ variable is instantiated
// per device by the runtime).
__device__ unsigned g_dev_status;

}  // namespace

unsigned *device_status_ptr() {
    static std::mutex mu;
    static unsigned *ptrs[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dev_status) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<unsigned *>(p);
    }
    return ptrs[dev];
}

// The chain workspace pool of the current device: a library-owned memory pool
// whose release threshold keeps freed blocks for the next call (so a chain
// call does not map and unmap its workspace every time), or nullptr.
cudaMemPool_t chain_pool() {
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
        uint64_t keep = UINT64_MAX;
        if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) {
            (void)cudaMemPoolDestroy(pool);
            return nullptr;
        }
        pools[dev] = pool;
    }
    return pools[dev];
}

namespace {
std::atomic<long long> g_pool_allocs{0};  // successful pool_alloc calls, all devices
}  // namespace

// KS_FAULT_INJECT=alloc: every workspace allocation fails (tests of the
// KS_ERR_ALLOC paths).
bool inject_alloc_failure() {
    const char *f = getenv("KS_FAULT_INJECT");
    return f && strcmp(f, "alloc") == 0;
}

cudaError_t pool_alloc(void **ptr, size_t bytes, cudaStream_t stream) {
    if (inject_alloc_failure()) return cudaErrorMemoryAllocation;
    cudaMemPool_t pool = chain_pool();
    if (!pool) {
        (void)cudaGetLastError();
        return cudaErrorMemoryAllocation;
    }
    const cudaError_t e = cudaMallocFromPoolAsync(ptr, bytes, pool, stream);
    if (e == cudaSuccess) g_pool_allocs.fetch_add(1, std::memory_order_relaxed);
    return e;
}

int sm_count() {
    static std::mutex mu;
    static int counts[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lk(mu);
    if (!counts[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        counts[dev] = n;
    }
    return counts[dev];
}

ks_status record_error(ks_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return s;
}

ks_status matmul_no_workspace(const void *X, const void *V, int64_t a, int64_t b, int64_t c, int64_t d,
                              int64_t batch, void *Y, int dtype, void *stream) {
    Problem p;
    bool noop = false;
    ks_status s = make_problem(X, V, a, b, c, d, batch, Y, dtype, stream, &p, &noop);
    if (s != KS_OK || noop) return s;
    p.no_workspace = true;
    return run(p, KS_VARIANT_AUTO);
}

}  // namespace ks

using namespace ks;

extern "C" {

ks_status ks_matmul_variant(const void *X, const void *values, int64_t a, int64_t b, int64_t c,
                            int64_t d, int64_t batch, void *Y, int dtype, int variant, void *stream) {
    if (variant < KS_VARIANT_AUTO || variant > KS_VARIANT_TC)
        return fail(KS_ERR_INVALID_ARG, "unknown variant %d", variant);
    Problem p;
    bool noop = false;
    ks_status s = make_problem(X, values, a, b, c, d, batch, Y, dtype, stream, &p, &noop);
    if (s != KS_OK || noop) return s;
    return run(p, variant);
}

ks_status ks_matmul(const void *X, const void *values, int64_t a, int64_t b, int64_t c, int64_t d,
                    int64_t batch, void *Y, int dtype, void *stream) {
    return ks_matmul_variant(X, values, a, b, c, d, batch, Y, dtype, KS_VARIANT_AUTO, stream);
}

ks_status ks_matmul_ep(const void *X, const void *values, int64_t a, int64_t b, int64_t c, int64_t d,
                       int64_t batch, void *Y, int dtype, const void *bias, int activation, int variant,
                       void *stream) {
    if (variant < KS_VARIANT_AUTO || variant > KS_VARIANT_TC)
        return fail(KS_ERR_INVALID_ARG, "unknown variant %d", variant);
    if (activation < KS_ACT_NONE || activation > KS_ACT_GELU_ERF)
        return fail(KS_ERR_INVALID_ARG, "unknown activation %d", activation);
    Problem p;
    bool noop = false;
    ks_status s = make_problem(X, values, a, b, c, d, batch, Y, dtype, stream, &p, &noop);
    if (s != KS_OK || noop) return s;
    if (bias) {
        const int elem = p.elem_bytes();
        if ((s = check_align(bias, elem, "bias")) != KS_OK) return s;
        if (ranges_overlap(Y, batch * p.out_features() * elem, bias, p.out_features() * elem))
            return fail(KS_ERR_INVALID_ARG, "Y overlaps bias");
    }
    p.bias = bias;
    p.act = activation;
    return run(p, variant);
}

ks_status ks_plan(int64_t a, int64_t b, int64_t c, int64_t d, int64_t batch, int dtype, int *variant) {
    if (!variant) return fail(KS_ERR_INVALID_ARG, "variant must be non-null");
    ks_status s = check_dtype(dtype);
    if (s != KS_OK) return s;
    int64_t in_f = 0, out_f = 0, nvals = 0;
    if ((s = check_sizes(a, b, c, d, batch, &in_f, &out_f, &nvals)) != KS_OK) return s;
    // Assume 256-byte aligned buffers, as a fresh allocation has.
    static const char dummy[16] __attribute__((aligned(256))) = {};
    Problem p{dummy, dummy, (void *)(dummy + 0), a, b, c, d, std::max<int64_t>(batch, 1), dtype, nullptr};
    Plan plan;
    const char *why = "";
    if (!make_plan(p, KS_VARIANT_AUTO, &plan, &why))
        return fail(KS_ERR_UNSUPPORTED, "no kernel: %s", why);
    *variant = plan.variant;
    return KS_OK;
}

ks_status ks_chain(const void *X, const void *const *factors, const ks_pattern *patterns, int n_factors,
                   int64_t batch, void *Y, int dtype, void *stream) {
    return ks_chain_ex(X, factors, patterns, n_factors, batch, Y, dtype, 0, stream);
}

ks_status ks_chain_ex(const void *X, const void *const *factors, const ks_pattern *patterns, int n_factors,
                      int64_t batch, void *Y, int dtype, int flags, void *stream) {
    return ks_chain_ep(X, factors, patterns, n_factors, batch, Y, dtype, flags, nullptr, KS_ACT_NONE, stream);
}

ks_status ks_chain_ep(const void *X, const void *const *factors, const ks_pattern *patterns, int n_factors,
                      int64_t batch, void *Y, int dtype, int flags, const void *bias, int activation,
                      void *stream) {
    if (flags & ~KS_CHAIN_UNFUSED) return fail(KS_ERR_INVALID_ARG, "unknown chain flags 0x%x", flags);
    if (activation < KS_ACT_NONE || activation > KS_ACT_GELU_ERF)
        return fail(KS_ERR_INVALID_ARG, "unknown activation %d", activation);
    const bool has_ep = bias != nullptr || activation != KS_ACT_NONE;
    ks_status s = check_dtype(dtype);
    if (s != KS_OK) return s;
    if (n_factors <= 0 || !factors || !patterns)
        return fail(KS_ERR_INVALID_ARG, "need n_factors > 0 and non-null factors/patterns");
    int64_t widest = 0;
    for (int t = 0; t < n_factors; ++t) {
        const ks_pattern &q = patterns[t];
        int64_t in_f = 0, out_f = 0, nvals = 0;
        if ((s = check_sizes(q.a, q.b, q.c, q.d, batch, &in_f, &out_f, &nvals)) != KS_OK) {
            char tmp[512];
            snprintf(tmp, sizeof(tmp), "factor %d: %s", t, g_msg);
            return fail(s, "%s", tmp);
        }
        if (t > 0) {
            const ks_pattern &r = patterns[t - 1];
            if (r.a * r.b * r.d != in_f)
                return fail(KS_ERR_INVALID_ARG, "factor %d has input width %lld but factor %d outputs %lld", t,
                            (long long)in_f, t - 1, (long long)(r.a * r.b * r.d));
        }
        if (t < n_factors - 1) widest = std::max(widest, out_f);
        if (!factors[t]) return fail(KS_ERR_INVALID_ARG, "factor %d is null", t);
    }
    if (batch == 0) return KS_OK;
    if (!X || !Y) return fail(KS_ERR_INVALID_ARG, "X and Y must be non-null");
    const int elem = dtype == KS_BF16 ? 2 : 4;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n_factors == 1) {
        const ks_pattern &q = patterns[0];
        return ks_matmul_ep(X, factors[0], q.a, q.b, q.c, q.d, batch, Y, dtype, bias, activation, KS_VARIANT_AUTO, stream);
    }
    if (!(flags & KS_CHAIN_UNFUSED) && !has_ep && butterfly12_matches(patterns, n_factors)) {
        if ((s = check_align(X, elem, "X")) != KS_OK || (s = check_align(Y, elem, "Y")) != KS_OK) return s;
        for (int t = 0; t < n_factors; ++t)
            if ((s = check_align(factors[t], elem, "a factor")) != KS_OK) return s;
        const int64_t width = 4096 * (int64_t)elem * batch;
        if (ranges_overlap(Y, width, X, width)) return fail(KS_ERR_INVALID_ARG, "Y overlaps X");
        for (int t = 0; t < n_factors; ++t)
            if (ranges_overlap(Y, width, factors[t], 4096 * 2 * (int64_t)elem))
                return fail(KS_ERR_INVALID_ARG, "Y overlaps factor %d", t);
        if (butterfly12_supported(X, factors, Y, dtype)) {
            const cudaError_t e = launch_butterfly12(X, factors, batch, Y, dtype, st);
            if (e != cudaSuccess) return cuda_fail(e, "fused butterfly chain launch");
            return ok();
        }
    }
    // Two ping-pong intermediates in one stream-ordered allocation from the
    // library's pool (256-byte aligned halves).
    void *buf[2] = {nullptr, nullptr};
    const size_t bytes = ((size_t)batch * (size_t)widest * (size_t)elem + 255) / 256 * 256;
    const size_t total = n_factors > 2 ? 2 * bytes : bytes;
    {
        void *base = nullptr;
        cudaError_t e = pool_alloc(&base, total, st);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return fail(KS_ERR_ALLOC, "workspace allocation of %zu bytes failed: %s", total, cudaGetErrorString(e));
        }
        buf[0] = base;
        if (n_factors > 2) buf[1] = static_cast<char *>(base) + bytes;
    }
    const void *src = X;
    ks_status result = KS_OK;
    for (int t = 0; t < n_factors; ++t) {
        const ks_pattern &q = patterns[t];
        void *dst = (t == n_factors - 1) ? Y : buf[t & 1];
        result = (t == n_factors - 1)
                     ? ks_matmul_ep(src, factors[t], q.a, q.b, q.c, q.d, batch, dst, dtype, bias, activation,
                                    KS_VARIANT_AUTO, stream)
                     : ks_matmul(src, factors[t], q.a, q.b, q.c, q.d, batch, dst, dtype, stream);
        if (result != KS_OK) {
            char tmp[512];
            snprintf(tmp, sizeof(tmp), "factor %d: %s", t, g_msg);
            fail(result, "%s", tmp);
            break;
        }
        src = dst;
    }
    {
        cudaError_t e = cudaFreeAsync(buf[0], st);
        if (e != cudaSuccess && result == KS_OK) result = cuda_fail(e, "workspace free");
    }
    return result;
}

ks_status ks_matmul_dx(const void *dY, const void *values, int64_t a, int64_t b, int64_t c, int64_t d,
                       int64_t batch, void *dX, int dtype, void *stream) {
    ks_status s = check_dtype(dtype);
    if (s != KS_OK) return s;
    int64_t in_f = 0, out_f = 0, nvals = 0;
    if ((s = check_sizes(a, b, c, d, batch, &in_f, &out_f, &nvals)) != KS_OK) return s;
    if (batch == 0) return KS_OK;
    if (!dY || !values || !dX) return fail(KS_ERR_INVALID_ARG, "dY, values and dX must be non-null");
    const int elem = dtype == KS_BF16 ? 2 : 4;
    if ((s = check_align(dY, elem, "dY")) != KS_OK || (s = check_align(values, elem, "values")) != KS_OK ||
        (s = check_align(dX, elem, "dX")) != KS_OK)
        return s;
    if (ranges_overlap(dX, batch * in_f * elem, dY, batch * out_f * elem))
        return fail(KS_ERR_INVALID_ARG, "dX overlaps dY");
    if (ranges_overlap(dX, batch * in_f * elem, values, nvals * elem))
        return fail(KS_ERR_INVALID_ARG, "dX overlaps values");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *vt = nullptr;
    cudaError_t e = pool_alloc(&vt, (size_t)(nvals * elem), st);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return fail(KS_ERR_ALLOC, "workspace allocation of %lld bytes failed: %s", (long long)(nvals * elem),
                    cudaGetErrorString(e));
    }
    // dX = dY K is the KS product of pattern (a, c, b, d) with the blocks transposed.
    ks_status result = KS_OK;
    e = launch_transpose_blocks(values, vt, a * d, b, c, dtype, st);
    if (e != cudaSuccess) result = cuda_fail(e, "values transpose launch");
    if (result == KS_OK) {
        result = ks_matmul(dY, vt, a, c, b, d, batch, dX, dtype, stream);
        if (result != KS_OK) {
            char tmp[512];
            snprintf(tmp, sizeof(tmp), "dX product: %s", g_msg);
            fail(result, "%s", tmp);
        }
    }
    e = cudaFreeAsync(vt, st);
    if (e != cudaSuccess && result == KS_OK) result = cuda_fail(e, "workspace free");
    return result;
}

ks_status ks_matmul_dv(const void *dY, const void *X, int64_t a, int64_t b, int64_t c, int64_t d, int64_t batch,
                       void *dV, int dtype, void *stream) {
    ks_status s = check_dtype(dtype);
    if (s != KS_OK) return s;
    int64_t in_f = 0, out_f = 0, nvals = 0;
    if ((s = check_sizes(a, b, c, d, batch, &in_f, &out_f, &nvals)) != KS_OK) return s;
    if (!dV) return fail(KS_ERR_INVALID_ARG, "dV must be non-null");
    const int elem = dtype == KS_BF16 ? 2 : 4;
    if ((s = check_align(dV, elem, "dV")) != KS_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (batch == 0) {  // an empty sum
        cudaError_t e = cudaMemsetAsync(dV, 0, (size_t)(nvals * elem), st);
        return e == cudaSuccess ? ok() : cuda_fail(e, "dV clear");
    }
    if (!dY || !X) return fail(KS_ERR_INVALID_ARG, "dY and X must be non-null");
    if ((s = check_align(dY, elem, "dY")) != KS_OK || (s = check_align(X, elem, "X")) != KS_OK) return s;
    if (ranges_overlap(dV, nvals * elem, dY, batch * out_f * elem)) return fail(KS_ERR_INVALID_ARG, "dV overlaps dY");
    if (ranges_overlap(dV, nvals * elem, X, batch * in_f * elem)) return fail(KS_ERR_INVALID_ARG, "dV overlaps X");
    DvProblem q{dY, X, dV, a, b, c, d, batch, dtype, st};
    int splits = 1;
    long long rows_per_split = batch;
    dv_split(q, &splits, &rows_per_split);
    const size_t wbytes = (size_t)splits * (size_t)nvals * sizeof(float);
    void *w = nullptr;
    cudaError_t e = pool_alloc(&w, wbytes, st);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return fail(KS_ERR_ALLOC, "workspace allocation of %zu bytes failed: %s", wbytes, cudaGetErrorString(e));
    }
    ks_status result = KS_OK;
    e = launch_dv(q, static_cast<float *>(w), splits, rows_per_split);
    if (e != cudaSuccess) result = cuda_fail(e, "dV kernel launch");
    e = cudaFreeAsync(w, st);
    if (e != cudaSuccess && result == KS_OK) result = cuda_fail(e, "workspace free");
    return result == KS_OK ? ok() : result;
}

}  // extern "C"

namespace ks {
namespace {

// Three non-blocking streams per device for ks_matmul_host: host-to-device
// copies, products, device-to-host copies (created on first use, kept until
// the process exits).
cudaError_t host_streams(cudaStream_t (&out)[3]) {
    static std::mutex mu;
    static cudaStream_t streams[64][3] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    for (int k = 0; k < 3; ++k) {
        if (!streams[dev][k]) {
            e = cudaStreamCreateWithFlags(&streams[dev][k], cudaStreamNonBlocking);
            if (e != cudaSuccess) return e;
        }
        out[k] = streams[dev][k];
    }
    return cudaSuccess;
}

// Rows per chunk of a host-resident product (row_bytes = X plus Y per row,
// big_row_bytes = the larger of the two): n ~ sqrt(copy time of the larger
// direction / per-chunk cost) chunks, 1..32, since the pipeline's fill and
// drain cost about 1/n of the copies and each chunk a fixed ~15 us (launches,
// copy set-up); a multiple of 128 rows (the tensor-core tile), at most 256 MiB
// of X plus Y per buffer.  Measured against a fixed six chunks: 1.5x on a
// 10 MB product, 1.01-1.06x from 400 MB to 3.3 GB, mid sizes unchanged.
int64_t host_chunk_rows(int64_t batch, int64_t row_bytes, int64_t big_row_bytes) {
    const double t_us = (double)batch * (double)big_row_bytes / 50e3;  // at ~50 GB/s
    int64_t n = (int64_t)(std::sqrt(t_us / 15.0) + 0.5);
    n = std::max<int64_t>(1, std::min<int64_t>(32, n));
    int64_t r = (batch + n - 1) / n;
    r = (r + 127) / 128 * 128;
    const int64_t cap = std::max<int64_t>(128, ((int64_t)256 << 20) / std::max<int64_t>(row_bytes, 1) / 128 * 128);
    return std::min(std::min(r, cap), batch);
}

}  // namespace
}  // namespace ks

extern "C" {

ks_status ks_matmul_host(const void *X, const void *values, int64_t a, int64_t b, int64_t c, int64_t d, int64_t batch,
                         void *Y, int dtype, void *stream) {
    ks_status s = check_dtype(dtype);
    if (s != KS_OK) return s;
    int64_t in_f = 0, out_f = 0, nvals = 0;
    if ((s = check_sizes(a, b, c, d, batch, &in_f, &out_f, &nvals)) != KS_OK) return s;
    if (batch == 0) return KS_OK;
    if (!X || !values || !Y) return fail(KS_ERR_INVALID_ARG, "X, values and Y must be non-null");
    const int elem = dtype == KS_BF16 ? 2 : 4;
    if ((s = check_align(X, elem, "X")) != KS_OK || (s = check_align(values, elem, "values")) != KS_OK ||
        (s = check_align(Y, elem, "Y")) != KS_OK)
        return s;
    const int64_t ybytes = batch * out_f * elem;
    if (ranges_overlap(Y, ybytes, X, batch * in_f * elem)) return fail(KS_ERR_INVALID_ARG, "Y overlaps X");
    if (ranges_overlap(Y, ybytes, values, nvals * elem)) return fail(KS_ERR_INVALID_ARG, "Y overlaps values");
    cudaStream_t caller = static_cast<cudaStream_t>(stream);
    cudaStream_t st[3];
    cudaError_t e = host_streams(st);
    if (e != cudaSuccess) return cuda_fail(e, "creating the copy and product streams");
    const int64_t rows = host_chunk_rows(batch, (in_f + out_f) * elem, std::max(in_f, out_f) * elem);
    const int64_t n_chunks = (batch + rows - 1) / rows;
    const int nbuf = n_chunks > 1 ? 2 : 1;
    const size_t vbytes = ((size_t)(nvals * elem) + 255) / 256 * 256;
    const size_t xb = ((size_t)(rows * in_f * elem) + 255) / 256 * 256;
    const size_t yb = ((size_t)(rows * out_f * elem) + 255) / 256 * 256;
    char *dev = nullptr;
    e = pool_alloc(reinterpret_cast<void **>(&dev), vbytes + nbuf * (xb + yb), caller);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return fail(KS_ERR_ALLOC, "workspace allocation of %zu bytes failed: %s", vbytes + nbuf * (xb + yb),
                    cudaGetErrorString(e));
    }
    char *dv = dev, *dx[2] = {dev + vbytes, dev + vbytes + xb}, *dy[2] = {dev + vbytes + nbuf * xb,
                                                                         dev + vbytes + nbuf * xb + yb};
    // events: fork, and per buffer the last copy-in, product and copy-out on it
    cudaEvent_t ev[8] = {};
    ks_status result = KS_OK;
    for (int k = 0; k < 8 && result == KS_OK; ++k)
        if ((e = cudaEventCreateWithFlags(&ev[k], cudaEventDisableTiming)) != cudaSuccess)
            result = cuda_fail(e, "event create");
    cudaEvent_t fork = ev[0], vin = ev[1], in_done[2] = {ev[2], ev[3]}, cmp_done[2] = {ev[4], ev[5]},
                out_done[2] = {ev[6], ev[7]};
    auto chk = [&](cudaError_t err, const char *what) {
        if (err != cudaSuccess && result == KS_OK) result = cuda_fail(err, what);
        return result == KS_OK;
    };
    if (result == KS_OK && chk(cudaEventRecord(fork, caller), "event record")) {
        for (int k = 0; k < 3; ++k) chk(cudaStreamWaitEvent(st[k], fork, 0), "stream wait");
        chk(cudaMemcpyAsync(dv, values, (size_t)(nvals * elem), cudaMemcpyHostToDevice, st[0]), "values copy");
        chk(cudaEventRecord(vin, st[0]), "event record");
        chk(cudaStreamWaitEvent(st[1], vin, 0), "stream wait");
    }
    for (int64_t k = 0; k < n_chunks && result == KS_OK; ++k) {
        const int q = (int)(k % nbuf);
        const int64_t r0 = k * rows, nr = std::min(rows, batch - r0);
        // copy-in: the product of chunk k - 2 has finished reading dx[q]
        if (k >= nbuf) chk(cudaStreamWaitEvent(st[0], cmp_done[q], 0), "stream wait");
        chk(cudaMemcpyAsync(dx[q], static_cast<const char *>(X) + r0 * in_f * elem, (size_t)(nr * in_f * elem),
                            cudaMemcpyHostToDevice, st[0]),
            "X copy");
        chk(cudaEventRecord(in_done[q], st[0]), "event record");
        // product: its X has landed and the copy-out of chunk k - 2 has read dy[q]
        chk(cudaStreamWaitEvent(st[1], in_done[q], 0), "stream wait");
        if (k >= nbuf) chk(cudaStreamWaitEvent(st[1], out_done[q], 0), "stream wait");
        if (result != KS_OK) break;
        Problem p{dx[q], dv, dy[q], a, b, c, d, nr, dtype, st[1]};
        const ks_status r = run(p, KS_VARIANT_AUTO);
        if (r != KS_OK) {
            result = r;
            break;
        }
        chk(cudaEventRecord(cmp_done[q], st[1]), "event record");
        // copy-out
        chk(cudaStreamWaitEvent(st[2], cmp_done[q], 0), "stream wait");
        chk(cudaMemcpyAsync(static_cast<char *>(Y) + r0 * out_f * elem, dy[q], (size_t)(nr * out_f * elem),
                            cudaMemcpyDeviceToHost, st[2]),
            "Y copy");
        chk(cudaEventRecord(out_done[q], st[2]), "event record");
    }
    // join: the caller's stream waits for all three streams, then frees the workspace
    for (int k = 0; k < 3; ++k) {
        cudaEvent_t j = nullptr;
        if (cudaEventCreateWithFlags(&j, cudaEventDisableTiming) == cudaSuccess) {
            if (cudaEventRecord(j, st[k]) == cudaSuccess) (void)cudaStreamWaitEvent(caller, j, 0);
            (void)cudaEventDestroy(j);
        } else {
            (void)cudaGetLastError();
            (void)cudaStreamSynchronize(st[k]);
        }
    }
    e = cudaFreeAsync(dev, caller);
    if (e != cudaSuccess && result == KS_OK) result = cuda_fail(e, "workspace free");
    for (int k = 0; k < 8; ++k)
        if (ev[k]) (void)cudaEventDestroy(ev[k]);
    return result == KS_OK ? ok() : result;
}

ks_status ks_bias_grad(const void *dY, int64_t batch, int64_t width, void *db, int dtype, void *stream) {
    ks_status s = check_dtype(dtype);
    if (s != KS_OK) return s;
    if (batch < 0 || width <= 0) return fail(KS_ERR_INVALID_ARG, "need batch >= 0 and width > 0");
    int64_t cells = 0;
    if (!mul_ok(std::max<int64_t>(batch, 1), width, &cells) || !mul_ok(cells, 4, &cells))
        return fail(KS_ERR_INVALID_ARG, "sizes overflow int64");
    if (!db) return fail(KS_ERR_INVALID_ARG, "db must be non-null");
    const int elem = dtype == KS_BF16 ? 2 : 4;
    if ((s = check_align(db, elem, "db")) != KS_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (batch == 0) {  // an empty sum
        cudaError_t e = cudaMemsetAsync(db, 0, (size_t)(width * elem), st);
        return e == cudaSuccess ? ok() : cuda_fail(e, "db clear");
    }
    if (!dY) return fail(KS_ERR_INVALID_ARG, "dY must be non-null");
    if ((s = check_align(dY, elem, "dY")) != KS_OK) return s;
    if (ranges_overlap(db, width * elem, dY, batch * width * elem)) return fail(KS_ERR_INVALID_ARG, "db overlaps dY");
    int splits = 1;
    long long rows_per_split = batch;
    colsum_split(batch, width, &splits, &rows_per_split);
    const size_t wbytes = (size_t)splits * (size_t)width * sizeof(float);
    void *w = nullptr;
    cudaError_t e = pool_alloc(&w, wbytes, st);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return fail(KS_ERR_ALLOC, "workspace allocation of %zu bytes failed: %s", wbytes, cudaGetErrorString(e));
    }
    ks_status result = KS_OK;
    e = launch_colsum(dY, db, batch, width, dtype, static_cast<float *>(w), splits, rows_per_split, st);
    if (e != cudaSuccess) result = cuda_fail(e, "column-sum launch");
    e = cudaFreeAsync(w, st);
    if (e != cudaSuccess && result == KS_OK) result = cuda_fail(e, "workspace free");
    return result;
}

namespace {

// The product of butterfly factors F_p .. F_q of size 2^L (F_k = (2^(k-1), 2, 2, 2^(L-k))).
ks_pattern butterfly_range(int p, int q, int L) {
    return ks_pattern{1LL << (p - 1), 1LL << (q - p + 1), 1LL << (q - p + 1), 1LL << (L - q)};
}

// Splits the range [p, q], whose product values are P, in the middle and fits
// the two halves; recurses until single factors land in factors[k - 1].
ks_status factorize_range(const float *P, int p, int q, int L, float *const *factors, cudaStream_t st) {
    const int r = (p + q - 1) / 2;
    const ks_pattern p1 = butterfly_range(p, r, L), p2 = butterfly_range(r + 1, q, L);
    const int64_t n1 = p1.a * p1.b * p1.c * p1.d, n2 = p2.a * p2.b * p2.c * p2.d;
    float *v1 = nullptr, *v2 = nullptr;
    ks_status result = KS_OK;
    if (r == p) {
        v1 = factors[p - 1];
    } else if (pool_alloc(reinterpret_cast<void **>(&v1), (size_t)n1 * 4, st) != cudaSuccess) {
        (void)cudaGetLastError();
        return fail(KS_ERR_ALLOC, "factorization workspace of %lld bytes", (long long)(n1 * 4));
    }
    if (r + 1 == q) {
        v2 = factors[q - 1];
    } else if (pool_alloc(reinterpret_cast<void **>(&v2), (size_t)n2 * 4, st) != cudaSuccess) {
        (void)cudaGetLastError();
        result = fail(KS_ERR_ALLOC, "factorization workspace of %lld bytes", (long long)(n2 * 4));
    }
    if (result == KS_OK) {
        const cudaError_t e = launch_rank1_fit(P, v1, v2, p1.a, p1.b, p1.c, p2.b, p2.c, p2.d, st);
        if (e != cudaSuccess) result = cuda_fail(e, "rank-one fit launch");
    }
    if (result == KS_OK && r > p) result = factorize_range(v1, p, r, L, factors, st);
    if (result == KS_OK && q > r + 1) result = factorize_range(v2, r + 1, q, L, factors, st);
    if (r != p && v1) (void)cudaFreeAsync(v1, st);
    if (r + 1 != q && v2) (void)cudaFreeAsync(v2, st);
    return result;
}

}  // namespace

ks_status ks_butterfly_factorize(const void *A, int log2n, void *const *factors, int dtype, void *stream) {
    if (dtype != KS_F32 && dtype != KS_TF32)
        return fail(dtype == KS_BF16 ? KS_ERR_UNSUPPORTED : KS_ERR_INVALID_ARG,
                    "the factorization runs on fp32 matrices only (dtype %d)", dtype);
    if (log2n < 1 || log2n > 14) return fail(KS_ERR_INVALID_ARG, "log2n must be in 1..14 (got %d)", log2n);
    if (!A || !factors) return fail(KS_ERR_INVALID_ARG, "A and factors must be non-null");
    ks_status s;
    if ((s = check_align(A, 4, "A")) != KS_OK) return s;
    const int64_t N = 1LL << log2n;
    for (int k = 0; k < log2n; ++k) {
        if (!factors[k]) return fail(KS_ERR_INVALID_ARG, "factor %d is null", k);
        if ((s = check_align(factors[k], 4, "a factor")) != KS_OK) return s;
        if (ranges_overlap(factors[k], 2 * N * 4, A, N * N * 4)) return fail(KS_ERR_INVALID_ARG, "factor %d overlaps A", k);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (log2n == 1) {  // a single factor (1, 2, 2, 1) holds A itself
        const cudaError_t e = cudaMemcpyAsync(factors[0], A, 4 * 4, cudaMemcpyDeviceToDevice, st);
        return e == cudaSuccess ? ok() : cuda_fail(e, "copy");
    }
    float *const *f = reinterpret_cast<float *const *>(factors);
    const ks_status r = factorize_range(static_cast<const float *>(A), 1, log2n, log2n, f, st);
    return r == KS_OK ? ok() : r;
}

ks_status ks_workspace_info(int64_t *allocations, int64_t *reserved_bytes) {
    if (allocations) *allocations = g_pool_allocs.load(std::memory_order_relaxed);
    if (reserved_bytes) {
        *reserved_bytes = 0;
        cudaMemPool_t pool = chain_pool();
        if (!pool) {
            (void)cudaGetLastError();
            return fail(KS_ERR_CUDA, "workspace pool unavailable on this device");
        }
        uint64_t v = 0;
        const cudaError_t e = cudaMemPoolGetAttribute(pool, cudaMemPoolAttrReservedMemCurrent, &v);
        if (e != cudaSuccess) return cuda_fail(e, "reading the pool's reserved memory");
        *reserved_bytes = (int64_t)v;
    }
    return KS_OK;
}

const char *ks_last_error(void) { return g_msg; }

const char *ks_status_string(int status) {
    switch (status) {
        case KS_OK: return "KS_OK";
        case KS_ERR_INVALID_ARG: return "KS_ERR_INVALID_ARG";
        case KS_ERR_MISALIGNED: return "KS_ERR_MISALIGNED";
        case KS_ERR_UNSUPPORTED: return "KS_ERR_UNSUPPORTED";
        case KS_ERR_ALLOC: return "KS_ERR_ALLOC";
        case KS_ERR_CUDA: return "KS_ERR_CUDA";
        case KS_ERR_TIMEOUT: return "KS_ERR_TIMEOUT";
        default: return "KS_ERR_UNKNOWN";
    }
}

ks_status ks_sync_status(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    unsigned *p = device_status_ptr();
    if (!p) return fail(KS_ERR_CUDA, "device status word unavailable");
    unsigned v = 0;
    e = cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading device status");
    if (v != 0) {
        unsigned zero = 0;
        e = cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "clearing device status");
        if (v & kDevTimeout) return fail(KS_ERR_TIMEOUT, "a bounded device-side wait gave up (status 0x%x)", v);
        return fail(KS_ERR_CUDA, "device status 0x%x", v);
    }
    return KS_OK;
}

int ks_version(void) { return 100; }

}  // extern "C"
