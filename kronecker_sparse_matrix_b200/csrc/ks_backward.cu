// Gradients of a KS product Y = X K^T, for training the page's KSLinear layer
// (taxoreview.com page on Kronecker-sparse matrix multiplication, first
// abstract: the kernel ships as a PyTorch-compatible layer).
//
//   dX = dY K:   dX[n, i*c*d + j*d + l] = sum_k values[i, l, k, j] dY[n, i*b*d + k*d + l]
//                a KS product with pattern (a, c, b, d) whose blocks are the
//                transposes of the forward ones; run by transposing the values
//                (a*b*c*d elements, negligible next to the batch) and calling
//                the forward kernels.
//   dV:          dV[i, l, k, j] = sum_n dY[n, i*b*d + k*d + l] X[n, i*c*d + j*d + l]
//                for each (i, l) a (b x N) x (N x c) product, reduced over the
//                batch: dv_kernel below, split over row ranges, then a
//                reduction of the fp32 partial sums in a fixed order.
//   dbias:       db[col] = sum_n dY[n, col], the gradient of the layer's bias:
//                column sums over row ranges (colsum_kernel), reduced in the
//                same fixed order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdint>

#include "ks_internal.h"

namespace ks {
namespace {

__device__ __forceinline__ float ld_f(const float *p) { return __ldg(p); }
__device__ __forceinline__ float ld_f(const __nv_bfloat16 *p) { return __bfloat162float(p[0]); }
__device__ __forceinline__ void st_f(float *p, float v) { *p = v; }
// the VEC = 16 / sizeof(T) elements of one 16-byte unit, as floats
__device__ __forceinline__ void unpack16(const uint4 &w, float (&f)[4]) {
    f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y); f[2] = __uint_as_float(w.z); f[3] = __uint_as_float(w.w);
}
__device__ __forceinline__ void unpack16(const uint4 &w, float (&f)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u[h]));
        f[2 * h] = t.x;
        f[2 * h + 1] = t.y;
    }
}
__device__ __forceinline__ void st_f(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

// vt[i][l][j][k] = v[i][l][k][j]: 32 x 32 tiles of each b x c block through
// shared memory; one CTA of 32 x 8 threads per tile, tiles flattened over
// (block, k-tile, j-tile).
template <typename T>
__global__ void __launch_bounds__(256) transpose_blocks_kernel(const T *__restrict__ v, T *__restrict__ vt,
                                                               long long n_tiles, int b, int c, int tb, int tc) {
    __shared__ T tile[32][33];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (long long t = blockIdx.x; t < n_tiles; t += gridDim.x) {
        const long long blk = t / ((long long)tb * tc);
        const int r = (int)(t - blk * tb * tc);
        const int k0 = (r / tc) * 32, j0 = (r % tc) * 32;
        const T *src = v + blk * b * c;
        T *dst = vt + blk * b * c;
#pragma unroll
        for (int u = 0; u < 32; u += 8) {
            const int k = k0 + ty + u, j = j0 + tx;
            if (k < b && j < c) tile[ty + u][tx] = src[(long long)k * c + j];
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < 32; u += 8) {
            const int j = j0 + ty + u, k = k0 + tx;
            if (k < b && j < c) dst[(long long)j * b + k] = tile[tx][ty + u];
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// dv_kernel: one CTA per (block i, DL consecutive l, BK values of k, BJ values
// of j, row range).  Each warp owns one l and a 64 x 64 (k, j) piece; each
// thread 8 k x 16 j fp32 sums, updated per row n with fma.rn.f32x2 on pairs of
// j.  Stages of kNR rows of dY and X (the needed (k, l) and (j, l) runs) are
// staged through registers into shared memory as [n][l][k] and [n][l][j],
// the next stage's loads in flight while the current one computes.  With VEC
// (the DL values of l of one k or j are whole 16-byte units: bf16 with DL = 8,
// fp32 with DL = 4, 8, and 16-byte-aligned buffers) a thread loads 16-byte
// units; otherwise one element at a time.
constexpr int kDvThreads = 256;
constexpr int kNR = 8;  // rows per stage

template <int DL> struct DvShape;
template <> struct DvShape<8> { static constexpr int WPK = 1, WPJ = 1; };
template <> struct DvShape<4> { static constexpr int WPK = 2, WPJ = 1; };
template <> struct DvShape<2> { static constexpr int WPK = 2, WPJ = 2; };
template <> struct DvShape<1> { static constexpr int WPK = 4, WPJ = 2; };

template <int DL> struct DvTile {
    static constexpr int BK = 64 * DvShape<DL>::WPK, BJ = 64 * DvShape<DL>::WPJ;
    static constexpr int KP = BK + 4, JP = BJ + 4;          // padded row lengths
    static constexpr int SA = kNR * DL * KP, SB = kNR * DL * JP;  // floats per stage
    static constexpr int NA = (kNR * BK * DL + kDvThreads - 1) / kDvThreads;  // staged dY values per thread
    static constexpr int NB = (kNR * BJ * DL + kDvThreads - 1) / kDvThreads;
    static constexpr int SMEM = 2 * (SA + SB) * 4;
};

struct DvParams {
    const void *dY, *X;
    float *W;  // partial sums [split][a][d][b][c]
    long long N;
    int a, b, c, d;
    int in_f, out_f;
    int n_g, n_kb, n_jb;  // groups a*d/DL, k tiles, j tiles
    long long rows_per_split;
    long long vsize;      // a*b*c*d
};

template <typename T, int DL, bool VEC>
__global__ void __launch_bounds__(kDvThreads, 1) dv_kernel(const DvParams p) {
    using TL = DvTile<DL>;
    constexpr int BK = TL::BK, BJ = TL::BJ;
    constexpr int EV = 16 / (int)sizeof(T);  // elements per 16-byte unit
    constexpr int UPR = VEC ? DL / EV : 1;   // units per (row, k) or (row, j)
    // 16-byte units per thread and stage: e = (row, k, unit of l), unit fastest
    constexpr int NAV = VEC ? (kNR * BK * UPR + kDvThreads - 1) / kDvThreads : 1;
    constexpr int NBV = VEC ? (kNR * BJ * UPR + kDvThreads - 1) / kDvThreads : 1;
    extern __shared__ __align__(16) float dsm[];
    const T *dY = static_cast<const T *>(p.dY);
    const T *X = static_cast<const T *>(p.X);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int WPL = 8 / DL;  // warps per l
    const int w_l = warp / WPL, w_r = warp % WPL;
    const int kw = (w_r / DvShape<DL>::WPJ) * 64, jw = (w_r % DvShape<DL>::WPJ) * 64;
    const int lane_k = lane >> 2, lane_j = lane & 3;

    long long t = blockIdx.x;
    const int jb = (int)(t % p.n_jb); t /= p.n_jb;
    const int kb = (int)(t % p.n_kb); t /= p.n_kb;
    const int g = (int)(t % p.n_g);
    const long long split = t / p.n_g;
    const int gpi = p.d / DL;
    const int i = g / gpi, l0 = (g % gpi) * DL;
    const int k0 = kb * BK, j0 = jb * BJ;
    const long long n_begin = split * p.rows_per_split;
    const long long n_end = min(p.N, n_begin + p.rows_per_split);
    const int n_stages = (int)((n_end - n_begin + kNR - 1) / kNR);

    // staging roles: element e of a stage = (row, k or j, l), l fastest
    float ra[VEC ? 1 : TL::NA], rb[VEC ? 1 : TL::NB];
    uint4 va[NAV], vb[NBV];
    auto load_stage = [&](int s) {
        const long long nb = n_begin + (long long)s * kNR;
        if constexpr (VEC) {
#pragma unroll
            for (int u = 0; u < NAV; ++u) {
                const int e = tid + u * kDvThreads;
                const int lu = e % UPR, k = (e / UPR) % BK, r = e / (UPR * BK);
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (r < kNR && nb + r < n_end && k0 + k < p.b)
                    v = __ldg(reinterpret_cast<const uint4 *>(dY + (nb + r) * p.out_f + (long long)i * p.b * p.d +
                                                              (long long)(k0 + k) * p.d + l0 + lu * EV));
                va[u] = v;
            }
#pragma unroll
            for (int u = 0; u < NBV; ++u) {
                const int e = tid + u * kDvThreads;
                const int lu = e % UPR, j = (e / UPR) % BJ, r = e / (UPR * BJ);
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (r < kNR && nb + r < n_end && j0 + j < p.c)
                    v = __ldg(reinterpret_cast<const uint4 *>(X + (nb + r) * p.in_f + (long long)i * p.c * p.d +
                                                              (long long)(j0 + j) * p.d + l0 + lu * EV));
                vb[u] = v;
            }
        } else {
#pragma unroll
        for (int u = 0; u < TL::NA; ++u) {
            const int e = tid + u * kDvThreads;
            const int l = e % DL, k = (e / DL) % BK, r = e / (DL * BK);
            float v = 0.f;
            if (r < kNR && nb + r < n_end && k0 + k < p.b)
                v = ld_f(dY + (nb + r) * p.out_f + (long long)i * p.b * p.d + (long long)(k0 + k) * p.d + l0 + l);
            ra[u] = v;
        }
#pragma unroll
        for (int u = 0; u < TL::NB; ++u) {
            const int e = tid + u * kDvThreads;
            const int l = e % DL, j = (e / DL) % BJ, r = e / (DL * BJ);
            float v = 0.f;
            if (r < kNR && nb + r < n_end && j0 + j < p.c)
                v = ld_f(X + (nb + r) * p.in_f + (long long)i * p.c * p.d + (long long)(j0 + j) * p.d + l0 + l);
            rb[u] = v;
        }
        }
    };
    auto store_stage = [&](int buf) {
        float *sa = dsm + buf * (TL::SA + TL::SB);
        float *sb = sa + TL::SA;
        if constexpr (VEC) {
#pragma unroll
            for (int u = 0; u < NAV; ++u) {
                const int e = tid + u * kDvThreads;
                const int lu = e % UPR, k = (e / UPR) % BK, r = e / (UPR * BK);
                if (r < kNR) {
                    float f[EV];
                    unpack16(va[u], f);
#pragma unroll
                    for (int h = 0; h < EV; ++h) sa[(r * DL + lu * EV + h) * TL::KP + k] = f[h];
                }
            }
#pragma unroll
            for (int u = 0; u < NBV; ++u) {
                const int e = tid + u * kDvThreads;
                const int lu = e % UPR, j = (e / UPR) % BJ, r = e / (UPR * BJ);
                if (r < kNR) {
                    float f[EV];
                    unpack16(vb[u], f);
#pragma unroll
                    for (int h = 0; h < EV; ++h) sb[(r * DL + lu * EV + h) * TL::JP + j] = f[h];
                }
            }
        } else {
#pragma unroll
        for (int u = 0; u < TL::NA; ++u) {
            const int e = tid + u * kDvThreads;
            const int l = e % DL, k = (e / DL) % BK, r = e / (DL * BK);
            if (r < kNR) sa[(r * DL + l) * TL::KP + k] = ra[u];
        }
#pragma unroll
        for (int u = 0; u < TL::NB; ++u) {
            const int e = tid + u * kDvThreads;
            const int l = e % DL, j = (e / DL) % BJ, r = e / (DL * BJ);
            if (r < kNR) sb[(r * DL + l) * TL::JP + j] = rb[u];
        }
        }
    };

    // acc[m][2q + h]: k = k0 + kw + lane_k + 8m, j = j0 + jw + 4 lane_j + 16q + 2h + (0, 1)
    float2 acc[8][8];
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int h = 0; h < 8; ++h) acc[m][h] = make_float2(0.f, 0.f);

    if (n_stages > 0) {
        load_stage(0);
        store_stage(0);
    }
    __syncthreads();
    for (int s = 0; s < n_stages; ++s) {
        const int buf = s & 1;
        if (s + 1 < n_stages) load_stage(s + 1);  // in flight during this stage
        const float *sa = dsm + buf * (TL::SA + TL::SB);
        const float *sb = sa + TL::SA;
#pragma unroll
        for (int r = 0; r < kNR; ++r) {
            const float *ar = sa + (r * DL + w_l) * TL::KP + kw + lane_k;
            const float *br = sb + (r * DL + w_l) * TL::JP + jw + 4 * lane_j;
            float am[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) am[m] = ar[8 * m];
            float4 bq[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) bq[q] = *reinterpret_cast<const float4 *>(br + 16 * q);
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const float2 a2 = make_float2(am[m], am[m]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[m][2 * q] = __ffma2_rn(a2, make_float2(bq[q].x, bq[q].y), acc[m][2 * q]);
                    acc[m][2 * q + 1] = __ffma2_rn(a2, make_float2(bq[q].z, bq[q].w), acc[m][2 * q + 1]);
                }
            }
        }
        if (s + 1 < n_stages) store_stage(buf ^ 1);
        __syncthreads();
    }

    // partial sums of this row range, in the values layout
    float *w = p.W + split * p.vsize + ((long long)(i * p.d + l0 + w_l) * p.b) * p.c;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int k = k0 + kw + lane_k + 8 * m;
        if (k >= p.b) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = j0 + jw + 4 * lane_j + 16 * q + 2 * h;
                if (j < p.c) w[(long long)k * p.c + j] = acc[m][2 * q + h].x;
                if (j + 1 < p.c) w[(long long)k * p.c + j + 1] = acc[m][2 * q + h].y;
            }
    }
}

// dV[e] = sum over splits s = 0, 1, ... of W[s][e], rounded once to T.
template <typename T>
__global__ void __launch_bounds__(256) dv_reduce_kernel(const float *__restrict__ W, T *__restrict__ dV,
                                                        long long vsize, int splits) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < vsize; e += stride) {
        float acc = 0.f;
        for (int s = 0; s < splits; ++s) acc += W[(long long)s * vsize + e];
        st_f(dV + e, acc);
    }
}

template <typename T>
cudaError_t launch_dv_reduce(const DvProblem &q, float *W, int splits) {
    const long long vsize = q.a * q.b * q.c * q.d;
    const long long rb = std::min<long long>((vsize + 255) / 256, (long long)sm_count() * 8);
    dv_reduce_kernel<T><<<(int)std::max<long long>(rb, 1), 256, 0, q.stream>>>(W, static_cast<T *>(q.dV), vsize,
                                                                               splits);
    return cudaGetLastError();
}

template <typename T, int DL>
cudaError_t launch_dv_typed(const DvProblem &q, float *W, int splits, long long rows_per_split) {
    constexpr int EV = 16 / (int)sizeof(T);
    using TL = DvTile<DL>;
    DvParams p;
    p.dY = q.dY;
    p.X = q.X;
    p.W = W;
    p.N = q.batch;
    p.a = (int)q.a; p.b = (int)q.b; p.c = (int)q.c; p.d = (int)q.d;
    p.in_f = (int)(q.a * q.c * q.d);
    p.out_f = (int)(q.a * q.b * q.d);
    p.n_g = (int)(q.a * (q.d / DL));
    p.n_kb = (int)((q.b + TL::BK - 1) / TL::BK);
    p.n_jb = (int)((q.c + TL::BJ - 1) / TL::BJ);
    p.rows_per_split = rows_per_split;
    p.vsize = q.a * q.b * q.c * q.d;
    const long long grid = (long long)p.n_g * p.n_kb * p.n_jb * splits;
    if (grid > INT32_MAX) return cudaErrorInvalidConfiguration;
    const bool aligned = ((reinterpret_cast<uintptr_t>(q.dY) | reinterpret_cast<uintptr_t>(q.X)) % 16) == 0;
    auto kern = dv_kernel<T, DL, false>;
    if constexpr (DL % EV == 0)
        if (aligned) kern = dv_kernel<T, DL, true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TL::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<(int)grid, kDvThreads, TL::SMEM, q.stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_dv_reduce<T>(q, W, splits);
}

template <typename T>
cudaError_t launch_dv_dl(const DvProblem &q, float *W, int splits, long long rows_per_split) {
    switch (dv_dl(q.d)) {
        case 8: return launch_dv_typed<T, 8>(q, W, splits, rows_per_split);
        case 4: return launch_dv_typed<T, 4>(q, W, splits, rows_per_split);
        case 2: return launch_dv_typed<T, 2>(q, W, splits, rows_per_split);
        default: return launch_dv_typed<T, 1>(q, W, splits, rows_per_split);
    }
}

// Column sums of dY over one row range: thread = column (consecutive threads
// read consecutive columns of a row), blockIdx.y = range; fp32 sums in row
// order into W[range][col].
template <typename T>
__global__ void __launch_bounds__(256) colsum_kernel(const T *__restrict__ dY, float *__restrict__ W, long long N,
                                                     long long width, long long rows_per_split) {
    const long long col = (long long)blockIdx.x * 256 + threadIdx.x;
    if (col >= width) return;
    const long long r0 = (long long)blockIdx.y * rows_per_split;
    const long long r1 = min(N, r0 + rows_per_split);
    const T *p = dY + r0 * width + col;
    float s = 0.f;
    long long r = r0;
    for (; r + 4 <= r1; r += 4, p += 4 * width) {  // four independent loads in flight
        const float v0 = ld_f(p), v1 = ld_f(p + width), v2 = ld_f(p + 2 * width), v3 = ld_f(p + 3 * width);
        s += v0;
        s += v1;
        s += v2;
        s += v3;
    }
    for (; r < r1; ++r, p += width) s += ld_f(p);
    W[(long long)blockIdx.y * width + col] = s;
}

template <typename T>
__global__ void __launch_bounds__(256) colsum_reduce_kernel(const float *__restrict__ W, T *__restrict__ db,
                                                            long long width, int splits) {
    const long long col = (long long)blockIdx.x * 256 + threadIdx.x;
    if (col >= width) return;
    float s = 0.f;
    for (int k = 0; k < splits; ++k) s += W[(long long)k * width + col];
    st_f(db + col, s);
}

}  // namespace

void colsum_split(long long batch, long long width, int *splits, long long *rows_per_split) {
    const long long col_blocks = (width + 255) / 256;
    long long want = std::max<long long>(1, (4LL * sm_count() + col_blocks - 1) / col_blocks);
    want = std::min<long long>(want, std::max<long long>(1, batch / 64));  // at least 64 rows per range
    want = std::min<long long>(want, 65535);
    const long long rows = (batch + want - 1) / want;
    *rows_per_split = rows;
    *splits = (int)((batch + rows - 1) / rows);
}

cudaError_t launch_colsum(const void *dY, void *db, long long batch, long long width, int dtype, float *W, int splits,
                          long long rows_per_split, cudaStream_t stream) {
    const dim3 grid((unsigned)((width + 255) / 256), (unsigned)splits);
    const unsigned rgrid = (unsigned)((width + 255) / 256);
    if (dtype == KS_BF16) {
        colsum_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(dY), W, batch,
                                                                width, rows_per_split);
        colsum_reduce_kernel<__nv_bfloat16><<<rgrid, 256, 0, stream>>>(W, static_cast<__nv_bfloat16 *>(db), width,
                                                                      splits);
    } else {
        colsum_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float *>(dY), W, batch, width, rows_per_split);
        colsum_reduce_kernel<float><<<rgrid, 256, 0, stream>>>(W, static_cast<float *>(db), width, splits);
    }
    return cudaGetLastError();
}

int dv_dl(int64_t d) { return d % 8 == 0 ? 8 : d % 4 == 0 ? 4 : d % 2 == 0 ? 2 : 1; }

void dv_split(const DvProblem &q, int *splits, long long *rows_per_split) {
    if (dv_tc_supported(q)) {
        dv_tc_split(q, splits, rows_per_split);
        return;
    }
    const int dl = dv_dl(q.d);
    const int bk = 64 * (dl == 8 ? 1 : dl == 1 ? 4 : 2), bj = 64 * ((dl == 2 || dl == 1) ? 2 : 1);
    const long long tiles = q.a * (q.d / dl) * ((q.b + bk - 1) / bk) * ((q.c + bj - 1) / bj);
    const long long vsize = q.a * q.b * q.c * q.d;
    long long s = (2LL * sm_count() + tiles - 1) / tiles;
    s = std::min(s, std::max<long long>(1, q.batch / 64));                       // at least 64 rows each
    s = std::min(s, std::max<long long>(1, (256LL << 20) / (vsize * 4)));         // workspace <= 256 MiB
    s = std::max<long long>(1, std::min<long long>(s, 4096));
    const long long rps = (q.batch + s - 1) / s;
    *rows_per_split = rps;
    *splits = (int)((q.batch + rps - 1) / rps);
}

cudaError_t launch_dv(const DvProblem &q, float *W, int splits, long long rows_per_split) {
    if (dv_tc_supported(q)) {  // tensor cores for the partial sums, then the same ordered reduction
        cudaError_t e = launch_dv_tc(q, W, splits, rows_per_split);
        return e != cudaSuccess ? e : launch_dv_reduce<__nv_bfloat16>(q, W, splits);
    }
    if (q.dtype == KS_BF16) return launch_dv_dl<__nv_bfloat16>(q, W, splits, rows_per_split);
    return launch_dv_dl<float>(q, W, splits, rows_per_split);
}

cudaError_t launch_transpose_blocks(const void *v, void *vt, int64_t blocks, int64_t b, int64_t c, int dtype,
                                    cudaStream_t stream) {
    const int tb = (int)((b + 31) / 32), tc = (int)((c + 31) / 32);
    const long long n_tiles = blocks * tb * tc;
    const int grid = (int)std::max<long long>(1, std::min<long long>(n_tiles, (long long)sm_count() * 16));
    if (dtype == KS_BF16)
        transpose_blocks_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(v), static_cast<__nv_bfloat16 *>(vt), n_tiles, (int)b, (int)c, tb, tc);
    else
        transpose_blocks_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float *>(v),
                                                                 static_cast<float *>(vt), n_tiles, (int)b, (int)c,
                                                                 tb, tc);
    return cudaGetLastError();
}

}  // namespace ks
