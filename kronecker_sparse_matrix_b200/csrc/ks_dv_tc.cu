// dV on the tensor cores (bf16), the gradient of the page's KSLinear layer
// with respect to its values (taxoreview.com page on Kronecker-sparse matrix
// multiplication, first abstract: a PyTorch-compatible layer):
//
//   dV[i, l, k, j] = sum_n dY[n, i*b*d + k*d + l] * X[n, i*c*d + j*d + l]
//
// For one block i and offset l this is D_l[k, j] = sum_n A_l[k, n] B_l[j, n]:
// M = 128 values of k, N = c values of j, K = the batch rows, accumulated in
// fp32 in tensor memory.  A CTA takes one block i, 8 consecutive l (d % 8 ==
// 0), 128 k and a range of rows (a multiple of 16); its fp32 partial sums go
// to W[split][i][l][k][j] and dv_reduce_kernel (ks_backward.cu) adds the
// splits in a fixed order.
//
// Per stage of 16 rows n (one K step of kind::f16):
//   warp 0      one thread: TMA loads of dY viewed as (d, b, a, N), box (8 l,
//               128 k, 1, 16 n), and of X viewed as (d, c, a, N), box (8 l, c j,
//               1, 16 n); both land as [n][k or j][8 l] (k >= b and rows >= N
//               are zero-filled by the tensor maps);
//   warps 2..5  transpose both in place into per-l K-major planes with the
//               32-byte swizzle (the layout of the forward kernel's values
//               operand): row = one k or j, 32 bytes = the stage's 16 rows.  A
//               task is one k (or j) and 8 rows: it reads the 8 rows' 16-byte
//               units (8 l each), transposes 8 x 8 in registers and writes one
//               16-byte half-row per l; eight consecutive lanes take eight
//               consecutive k, so both the reads and the writes of a quarter-warp
//               reach eight bank groups;
//   warp 1      one thread issues per l one MMA (M = 128, N = c, K = 16) into
//               TMEM columns l*c .. l*c + c - 1.
// After the last stage warps 2..5 read the accumulators (warp w: TMEM lanes
// 32 (w % 4) ..) and store the partial sums.  Every mbarrier wait is bounded
// (about one second, or at once under KS_FAULT_INJECT=timeout); a wait that
// runs out sets the device status word and ends every role.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>

#include "ks_internal.h"
#include "ks_sm100.cuh"

namespace ks {
namespace {

using namespace sm100;

constexpr int kDvThreads = 192;  // 6 warps
constexpr int kDvStages = 3;
constexpr int kDvRows = 16;      // rows n per stage: one K step
constexpr int kDvM = 128;        // k per CTA (MMA M)
constexpr int kDvL = 8;          // l per CTA

struct DvTcParams {
    float *W;
    long long N, rows_per_split, vsize;
    int b, c, d;
    int n_g, n_kt;
    unsigned *status;
    unsigned long long wait_ns;  // bound of the pipeline's waits
};

__global__ void __launch_bounds__(kDvThreads, 1)
    dv_tc_kernel(const __grid_constant__ CUtensorMap ymap, const __grid_constant__ CUtensorMap xmap, const DvTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int c = p.c;
    const int a_bytes = kDvRows * kDvM * 16;  // 32 KB: raw [n][k][8 l], then 8 planes of 128 rows x 32 B
    const int b_bytes = kDvRows * c * 16;     // raw [n][j][8 l], then 8 planes of c rows x 32 B
    const int stage_bytes = a_bytes + b_bytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kDvStages * stage_bytes);
    uint64_t *x_full = bars;                  // [kDvStages] TMA landed
    uint64_t *a_ready = x_full + kDvStages;   // [kDvStages] transposed
    uint64_t *x_empty = a_ready + kDvStages;  // [kDvStages] MMAs done with it
    uint64_t *done = x_empty + kDvStages;     // [1] every MMA done
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long t = blockIdx.x;
    const int kt = (int)(t % p.n_kt); t /= p.n_kt;
    const int g = (int)(t % p.n_g);
    const long long split = t / p.n_g;
    const int gpi = p.d / kDvL;
    const int i = g / gpi, l0 = (g % gpi) * kDvL;
    const int k0 = kt * kDvM;
    const long long n_begin = split * p.rows_per_split;
    const long long n_end = min(p.N, n_begin + p.rows_per_split);
    const int n_stages = (int)((n_end - n_begin + kDvRows - 1) / kDvRows);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDvStages; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&a_ready[s], 128);
            mbar_init(&x_empty[s], 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(tmem_holder, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (one thread)
        if (lane == 0) {
            bool ok = true;
            int s = 0;
            for (; s < n_stages && ok; ++s) {
                const int slot = s % kDvStages;
                ok = mbar_wait(&x_empty[slot], ((s / kDvStages) & 1) ^ 1, abort_flag, p.status, p.wait_ns);
                if (!ok) break;
                uint8_t *st = smem + slot * stage_bytes;
                const int n0 = (int)(n_begin + (long long)s * kDvRows);
                mbar_expect_tx(&x_full[slot], (uint32_t)stage_bytes);
                tma_load_4d(st, &ymap, &x_full[slot], l0, k0, i, n0);
                tma_load_4d(st + a_bytes, &xmap, &x_full[slot], l0, 0, i, n0);
            }
            // on abort, copies already issued may still be landing: wait (bounded) for them
            if (*abort_flag)
                for (int k = std::max(0, s - kDvStages); k < s; ++k) mbar_wait_drain(&x_full[k % kDvStages], (k / kDvStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (one thread)
        if (lane == 0) {
            // D fp32 (bit 4); A and B bf16 (format 1, bits 7 and 10), both
            // K-major; N = c (bits 17-22, N / 8), M = 128 (bits 24-28, M / 16)
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(c >> 3) << 17) |
                                   ((uint32_t)(kDvM >> 4) << 24);
            bool ok = true;
            for (int s = 0; s < n_stages && ok; ++s) {
                const int slot = s % kDvStages;
                ok = mbar_wait(&a_ready[slot], (s / kDvStages) & 1, abort_flag, p.status, p.wait_ns);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sa = su32(smem + slot * stage_bytes), sb = sa + (uint32_t)a_bytes;
#pragma unroll
                for (int l = 0; l < kDvL; ++l) {
                    const uint64_t ad = smem_desc_sw(sa + (uint32_t)(l * kDvM * 32), 256, 6u);
                    const uint64_t bd = smem_desc_sw(sb + (uint32_t)(l * c * 32), 256, 6u);
                    mma_bf16(tmem_base + (uint32_t)(l * c), ad, bd, idesc, s > 0 ? 1u : 0u);
                }
                mma_commit(&x_empty[slot]);
            }
            mma_commit(done);  // fires when every MMA issued above has finished
        }
    } else {
        // ------------------------------------------------ transpose, then epilogue (warps 2..5)
        const int tt = threadIdx.x - 64;  // 0..127
        bool ok = true;
        for (int s = 0; s < n_stages && ok; ++s) {
            const int slot = s % kDvStages;
            const bool w = mbar_wait(&x_full[slot], (s / kDvStages) & 1, abort_flag, p.status, p.wait_ns);
            ok = bar_and(1, 128, w);  // uniform over the four warps
            if (!ok) break;
            uint8_t *st = smem + slot * stage_bytes;
            // A: tasks (k = tt, row half nh = 0, 1); B: task (j = tt % c, nh = tt / c) for tt < 2c
            uint4 oa[2][8], ob[8];
#pragma unroll
            for (int nh = 0; nh < 2; ++nh) {
                uint4 in[8];
#pragma unroll
                for (int r = 0; r < 8; ++r)
                    in[r] = *reinterpret_cast<const uint4 *>(st + ((8 * nh + r) * kDvM + tt) * 16);
                transpose8x8_b16(in, oa[nh]);
            }
            const bool has_b = tt < 2 * c;
            const int jb = has_b ? tt % c : 0, nb = has_b ? tt / c : 0;
            if (has_b) {
                uint4 in[8];
#pragma unroll
                for (int r = 0; r < 8; ++r)
                    in[r] = *reinterpret_cast<const uint4 *>(st + a_bytes + ((8 * nb + r) * c + jb) * 16);
                transpose8x8_b16(in, ob);
            }
            bar_sync(1, 128);  // every read of the raw stage is done
            // plane l, row m: 32 bytes at l * rows * 32 + m * 32, half h at h ^ bit 2 of m
#pragma unroll
            for (int nh = 0; nh < 2; ++nh)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    *reinterpret_cast<uint4 *>(st + e * kDvM * 32 + tt * 32 + ((nh ^ ((tt >> 2) & 1)) << 4)) = oa[nh][e];
            if (has_b) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    *reinterpret_cast<uint4 *>(st + a_bytes + e * c * 32 + jb * 32 + ((nb ^ ((jb >> 2) & 1)) << 4)) = ob[e];
            }
            fence_proxy_async();
            mbar_arrive(&a_ready[slot]);
        }
        // epilogue: this warp's 32 TMEM lanes are k = k0 + 32 (warp % 4) + lane
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(done, 0, abort_flag, p.status, p.wait_ns));
        if (ok && n_stages > 0) {
            tc_fence_after();
            const int quad = warp & 3;
            const int k = k0 + 32 * quad + lane;
            float *wrow = p.W + split * p.vsize + ((long long)(i * p.d + l0) * p.b + k) * c;
            const long long lstride = (long long)p.b * c;  // next l
            for (int l = 0; l < kDvL; ++l) {
                for (int j8 = 0; j8 < c; j8 += 8) {
                    float v[8];
                    tmem_ld8(tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(l * c + j8), v);
                    tmem_ld_wait();
                    if (k < p.b) {
                        float4 *dst = reinterpret_cast<float4 *>(wrow + l * lstride + j8);
                        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        // every MMA issued has finished before TMEM is freed (done may already have fired)
        if (lane == 0 && *abort_flag) mbar_wait_drain(done, 0);
        __syncwarp();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace

// bf16, d % 8 == 0, c a multiple of 16 up to 64 (8 l x c TMEM columns <= 512),
// b >= 128 (the dY box spans 128 k) and 16-byte-aligned buffers.
bool dv_tc_supported(const DvProblem &q) {
    if (q.dtype != KS_BF16 || q.d % 8 || q.c % 16 || q.c > 64 || q.b < kDvM) return false;
    if (((reinterpret_cast<uintptr_t>(q.dY) | reinterpret_cast<uintptr_t>(q.X)) % 16) != 0) return false;
    if (q.batch > (1LL << 31) - 256 || q.a * q.d > (1LL << 31) || q.a > 65535) return false;
    return tensor_map_encoder() != nullptr;
}

// Row ranges (multiples of 16) so that the CTAs fill the SMs about once.
void dv_tc_split(const DvProblem &q, int *splits, long long *rows_per_split) {
    const long long tiles = (q.a * (q.d / kDvL)) * ((q.b + kDvM - 1) / kDvM);
    const long long max_splits = (q.batch + kDvRows - 1) / kDvRows;
    const long long vsize = q.a * q.b * q.c * q.d;
    long long s = std::min<long long>(max_splits, (long long)sm_count() / std::max<long long>(1, tiles));
    s = std::max<long long>(1, std::min<long long>(s, (256LL << 20) / (vsize * 4)));  // workspace <= 256 MiB
    long long rows = ((q.batch + s - 1) / s + kDvRows - 1) / kDvRows * kDvRows;
    s = (q.batch + rows - 1) / rows;
    *splits = (int)s;
    *rows_per_split = rows;
}

cudaError_t launch_dv_tc(const DvProblem &q, float *W, int splits, long long rows_per_split) {
    auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
    if (!encode || rows_per_split % kDvRows) return cudaErrorInvalidConfiguration;
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUtensorMap ymap, xmap;
    {
        // dY as (d, b, a, N): a box (8 l, 128 k, 1, 16 rows)
        cuuint64_t dims[4] = {(cuuint64_t)q.d, (cuuint64_t)q.b, (cuuint64_t)q.a, (cuuint64_t)q.batch};
        cuuint64_t strides[3] = {(cuuint64_t)q.d * 2, (cuuint64_t)q.b * q.d * 2, (cuuint64_t)q.a * q.b * q.d * 2};
        cuuint32_t box[4] = {(cuuint32_t)kDvL, (cuuint32_t)kDvM, 1, (cuuint32_t)kDvRows};
        if (encode(&ymap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(q.dY), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        // X as (d, c, a, N): a box (8 l, c j, 1, 16 rows)
        cuuint64_t dims[4] = {(cuuint64_t)q.d, (cuuint64_t)q.c, (cuuint64_t)q.a, (cuuint64_t)q.batch};
        cuuint64_t strides[3] = {(cuuint64_t)q.d * 2, (cuuint64_t)q.c * q.d * 2, (cuuint64_t)q.a * q.c * q.d * 2};
        cuuint32_t box[4] = {(cuuint32_t)kDvL, (cuuint32_t)q.c, 1, (cuuint32_t)kDvRows};
        if (encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(q.X), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    DvTcParams p;
    p.W = W;
    p.N = q.batch;
    p.rows_per_split = rows_per_split;
    p.vsize = q.a * q.b * q.c * q.d;
    p.b = (int)q.b;
    p.c = (int)q.c;
    p.d = (int)q.d;
    p.n_g = (int)(q.a * (q.d / kDvL));
    p.n_kt = (int)((q.b + kDvM - 1) / kDvM);
    p.status = device_status_ptr();
    if (!p.status) return cudaErrorUnknown;
    p.wait_ns = pipeline_wait_bound_ns();
    const int stage_bytes = kDvRows * (kDvM + (int)q.c) * 16;
    const int smem = kDvStages * stage_bytes + 3 * kDvStages * 8 + 8 + 16 + 1024;
    const long long grid = (long long)p.n_g * p.n_kt * splits;
    if (grid > INT32_MAX) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(dv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dv_tc_kernel<<<(int)grid, kDvThreads, smem, q.stream>>>(ymap, xmap, p);
    return cudaGetLastError();
}

}  // namespace ks
