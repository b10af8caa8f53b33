// Output-stationary CUDA-core gather-GEMM for one KS factor, register-staged
// (bf16, and fp32 problems beyond the cp.async kernel's 32-bit tile index).
//
// Y[n, i*b*d + k*d + l] = sum_{j<c} values[i, l, k, j] * X[n, i*c*d + j*d + l]
// (taxoreview.com page on Kronecker-sparse matrix multiplication, first
// abstract: a fused, output-stationary kernel with no permutation passes).
//
// For a fixed block i and offset l the product is a dense GEMM
//     Y_il[n, k] = sum_j X_il[n, j] * V_il[k, j],
// whose A operand X_il is X's columns i*c*d + j*d + l: a stride-d gather.
// One 32-byte sector of X holds 8 consecutive l (fp32), so a CTA takes DL
// consecutive l at once (DL = min(d, 8)) and every byte it pulls from L2 is
// used.  A CTA tile is (BM rows) x (BKL values of k) x (DL values of l) for one
// block i, accumulated in registers over the whole reduction j < c:
//
//  * stage loads: for JT = 8 values of j, 16-byte loads of X rows (runs of DL
//    contiguous l, or one run of JT*d when DL == d) and of values (runs of
//    consecutive j), kept in registers while the previous stage computes, then
//    written transposed to shared memory as As[l][j][n] and Bs[l][j][k];
//  * compute: each warp owns one l and a 64 x (4*TN) piece of (n, k); each
//    thread an 8 x TN register tile, updated with packed fp32x2 FMAs
//    (fma.rn.f32x2, two FMAs per issue slot on sm_100), operands read as
//    float4 from shared memory;
//  * epilogue: accumulators go through shared memory in [n][l][k] order and
//    leave as 16-byte coalesced stores of Y[n, i, k, l-run].
//
// Rounding: every product and sum is an fp32 fma.rn; the order is j = 0..c-1
// per output, the same as a scalar loop.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "ks_epilogue.cuh"
#include "ks_internal.h"

namespace ks {
namespace {

constexpr int kThreads = 256;
constexpr int kJT = 8;  // j per stage
constexpr int kTM = 8;  // rows per thread

struct FmaParams {
    const void *X;
    const void *V;
    void *Y;
    const void *bias;  // fused epilogue: out_f values of T, or null
    int act;
    long long N;
    int a, b, c, d;
    int in_f, out_f;
    int n_rb, n_g, n_kb;  // row blocks, (i, l-group) groups, k blocks
    long long n_tiles;
};

template <typename T> struct Elem;
template <> struct Elem<float> {
    static constexpr int E = 4;  // elements per 16 bytes
    __device__ static void unpack(const uint4 &u, float (&v)[4]) {
        v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
        v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
    }
    __device__ static uint4 pack(const float (&v)[4]) {
        return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
    }
};
template <> struct Elem<__nv_bfloat16> {
    static constexpr int E = 8;
    __device__ static void unpack(const uint4 &u, float (&v)[8]) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            v[2 * q] = __uint_as_float(w[q] << 16);
            v[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
        }
    }
    __device__ static uint4 pack(const float (&v)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
            w[q] = *reinterpret_cast<uint32_t *>(&h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <int DL, int WM, int WK, int TN>
struct Tile {
    static_assert(DL * WM * WK == 8, "8 warps per CTA");
    static_assert(TN % 4 == 0 && TN >= 8 && TN <= 16, "thread tile k");
    static constexpr int BM = 64 * WM;
    static constexpr int BKL = 4 * TN * WK;
    static constexpr int BMP = BM + 4;            // As row stride (floats)
    static constexpr int PSA = kJT * BMP + 4;      // As plane (l) stride, = 4 mod 8
    static constexpr int BKP = BKL + 4;           // Bs row stride, = 4 mod 8
    static constexpr int PSB = kJT * BKP + 4;      // Bs plane stride
    static constexpr int STAGE = DL * (PSA + PSB); // floats per pipeline buffer
    static constexpr int RS = DL * BKP + (DL == 1 ? 0 : 4);  // epilogue row stride, = 4 mod 8
    static constexpr int EPI = (BM / 2) * RS;      // epilogue floats (half the rows at a time)
    static constexpr int SMEM_FLOATS = (2 * STAGE > EPI) ? 2 * STAGE : EPI;
};

template <typename T, int DL, int WM, int WK, int TN>
__global__ void __launch_bounds__(kThreads, 1) fma_kernel(const FmaParams p) {
    using TL = Tile<DL, WM, WK, TN>;
    constexpr int E = Elem<T>::E;
    constexpr int BM = TL::BM, BKL = TL::BKL;
    constexpr int UX = kJT * DL / E;                 // 16-byte units of X per row per stage
    constexpr int UG = UX < 8 ? UX : 8;              // units per lane group
    constexpr int NX = (BM * UX + kThreads - 1) / kThreads;
    constexpr int JQ = kJT / E > 0 ? kJT / E : 1;    // 16-byte units of values per (l, k) per stage
    constexpr int NV = (DL * BKL * JQ + kThreads - 1) / kThreads;
    constexpr int UO = BKL * DL / E;                 // 16-byte output units per row
    static_assert(kJT % E == 0 || E == 8, "stage covers whole 16-byte value units");

    extern __shared__ __align__(16) float smem[];

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int w_l = warp / (WM * WK);
    const int w_m = (warp / WK) % WM;
    const int w_k = warp % WK;
    const int lane_r = lane >> 2, lane_k = lane & 3;

    const T *__restrict__ X = static_cast<const T *>(p.X);
    const T *__restrict__ V = static_cast<const T *>(p.V);
    T *__restrict__ Y = static_cast<T *>(p.Y);
    const int n_stages = (p.c + kJT - 1) / kJT;
    const int groups_per_i = p.d / DL;

    for (long long tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x) {
        const int kb = (int)(tile % p.n_kb);
        const long long rest = tile / p.n_kb;
        const int g = (int)(rest % p.n_g);
        const int rb = (int)(rest / p.n_g);
        const int i = g / groups_per_i;
        const int l0 = (g % groups_per_i) * DL;
        const long long n0 = (long long)rb * BM;
        const int k0 = kb * BKL;

        const T *x_tile = X + n0 * p.in_f + (long long)i * p.c * p.d + l0;
        const T *v_tile = V + ((long long)i * p.d + l0) * p.b * p.c;

        uint4 rx[NX], rv[NV];

        auto load_stage = [&](int s) {
            const int j0 = s * kJT;
#pragma unroll
            for (int t = 0; t < NX; ++t) {
                const int idx = tid + t * kThreads;
                const int u_lo = idx % UG;
                const int rest2 = idx / UG;
                const int r = rest2 % BM;
                const int u = (rest2 / BM) * UG + u_lo;
                const int f = u * E;                  // flat (j_local, l_local) element
                const int jl = f / DL, ll = f % DL;
                rx[t] = make_uint4(0, 0, 0, 0);
                if (idx < BM * UX && n0 + r < p.N && j0 + jl < p.c) {
                    const T *src = x_tile + (long long)r * p.in_f + (long long)(j0 + jl) * p.d + ll;
                    rx[t] = __ldg(reinterpret_cast<const uint4 *>(src));
                }
            }
#pragma unroll
            for (int t = 0; t < NV; ++t) {
                const int idx = tid + t * kThreads;
                const int jq = idx % JQ;
                const int rest2 = idx / JQ;
                const int kl = rest2 % BKL;
                const int ll = rest2 / BKL;
                const int j = j0 + jq * E;
                rv[t] = make_uint4(0, 0, 0, 0);
                if (idx < DL * BKL * JQ && k0 + kl < p.b && j < p.c) {
                    const T *src = v_tile + ((long long)ll * p.b + (k0 + kl)) * p.c + j;
                    rv[t] = __ldg(reinterpret_cast<const uint4 *>(src));
                }
            }
        };

        auto store_stage = [&](int buf) {
            float *As = smem + buf * TL::STAGE;
            float *Bs = As + DL * TL::PSA;
#pragma unroll
            for (int t = 0; t < NX; ++t) {
                const int idx = tid + t * kThreads;
                if (idx < BM * UX) {
                    const int u_lo = idx % UG;
                    const int rest2 = idx / UG;
                    const int r = rest2 % BM;
                    const int u = (rest2 / BM) * UG + u_lo;
                    float v[E];
                    Elem<T>::unpack(rx[t], v);
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const int f = u * E + e;
                        const int jl = f / DL, ll = f % DL;
                        As[ll * TL::PSA + jl * TL::BMP + r] = v[e];
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < NV; ++t) {
                const int idx = tid + t * kThreads;
                if (idx < DL * BKL * JQ) {
                    const int jq = idx % JQ;
                    const int rest2 = idx / JQ;
                    const int kl = rest2 % BKL;
                    const int ll = rest2 / BKL;
                    float v[E];
                    Elem<T>::unpack(rv[t], v);
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const int jl = jq * E + e;
                        if (jl < kJT) Bs[ll * TL::PSB + jl * TL::BKP + kl] = v[e];
                    }
                }
            }
        };

        float2 acc[kTM][TN / 2];
#pragma unroll
        for (int m = 0; m < kTM; ++m)
#pragma unroll
            for (int q = 0; q < TN / 2; ++q) acc[m][q] = make_float2(0.f, 0.f);

        load_stage(0);
        store_stage(0);
        __syncthreads();

        for (int s = 0; s < n_stages; ++s) {
            const int buf = s & 1;
            if (s + 1 < n_stages) load_stage(s + 1);
            const float *As = smem + buf * TL::STAGE + w_l * TL::PSA + w_m * 64 + lane_r * 4;
            const float *Bs = smem + buf * TL::STAGE + DL * TL::PSA + w_l * TL::PSB + w_k * (4 * TN) + lane_k * 4;
#pragma unroll
            for (int jj = 0; jj < kJT; ++jj) {
                const float4 a0 = *reinterpret_cast<const float4 *>(As + jj * TL::BMP);
                const float4 a1 = *reinterpret_cast<const float4 *>(As + jj * TL::BMP + 32);
                float4 bq[TN / 4];
#pragma unroll
                for (int q = 0; q < TN / 4; ++q) bq[q] = *reinterpret_cast<const float4 *>(Bs + jj * TL::BKP + 16 * q);
                const float am[kTM] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                for (int m = 0; m < kTM; ++m) {
                    const float2 a2 = make_float2(am[m], am[m]);
#pragma unroll
                    for (int q = 0; q < TN / 4; ++q) {
                        acc[m][2 * q] = __ffma2_rn(a2, make_float2(bq[q].x, bq[q].y), acc[m][2 * q]);
                        acc[m][2 * q + 1] = __ffma2_rn(a2, make_float2(bq[q].z, bq[q].w), acc[m][2 * q + 1]);
                    }
                }
            }
            if (s + 1 < n_stages) store_stage(buf ^ 1);
            __syncthreads();
        }

        // Epilogue, half of the rows at a time: Cs[rr][l][k], rr = w_m*32 + lane_r*4 + mm.
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float *Cs = smem;
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
                const int m = 4 * h + mm;
                const int rr = w_m * 32 + lane_r * 4 + mm;
                float *dst = Cs + rr * TL::RS + w_l * TL::BKP + w_k * (4 * TN) + lane_k * 4;
#pragma unroll
                for (int q = 0; q < TN / 4; ++q)
                    *reinterpret_cast<float4 *>(dst + 16 * q) =
                        make_float4(acc[m][2 * q].x, acc[m][2 * q].y, acc[m][2 * q + 1].x, acc[m][2 * q + 1].y);
            }
            __syncthreads();
            for (int idx = tid; idx < (BM / 2) * UO; idx += kThreads) {
                const int rr = idx / UO;
                const int uo = idx % UO;
                const long long row = n0 + (rr / 32) * 64 + 32 * h + (rr % 32);
                const int f = uo * E;                 // flat (k_local, l_local)
                const int kl = f / DL, ll = f % DL;
                if (row < p.N && k0 + kl < p.b) {
                    float v[E];
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const int fe = f + e;
                        v[e] = Cs[rr * TL::RS + (fe % DL) * TL::BKP + fe / DL];
                    }
                    const long long col = (long long)i * p.b * p.d + (long long)(k0 + kl) * p.d + l0 + ll;
                    if (p.bias) {
#pragma unroll
                        for (int e = 0; e < E; ++e) v[e] += ep_bias(static_cast<const T *>(p.bias), col + e);
                    }
                    if (p.act) ep_act_array(v, p.act);
                    *reinterpret_cast<uint4 *>(Y + row * p.out_f + col) = Elem<T>::pack(v);
                }
            }
            __syncthreads();
        }
    }
}

template <typename T, int DL, int WM, int WK, int TN>
cudaError_t launch_cfg(const Problem &pr) {
    using TL = Tile<DL, WM, WK, TN>;
    FmaParams p;
    p.X = pr.X;
    p.V = pr.V;
    p.Y = pr.Y;
    p.bias = pr.bias;
    p.act = pr.act;
    p.N = pr.batch;
    p.a = (int)pr.a; p.b = (int)pr.b; p.c = (int)pr.c; p.d = (int)pr.d;
    p.in_f = (int)pr.in_features();
    p.out_f = (int)pr.out_features();
    p.n_rb = (int)((pr.batch + TL::BM - 1) / TL::BM);
    p.n_g = (int)(pr.a * (pr.d / DL));
    p.n_kb = (int)((pr.b + TL::BKL - 1) / TL::BKL);
    p.n_tiles = (long long)p.n_rb * p.n_g * p.n_kb;
    const size_t smem = (size_t)TL::SMEM_FLOATS * sizeof(float);
    auto kern = fma_kernel<T, DL, WM, WK, TN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = std::min<long long>(p.n_tiles, (long long)sm_count());
    kern<<<(int)grid, kThreads, smem, pr.stream>>>(p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const Problem &p, const FmaConfig &c) {
#define KS_FMA_CASE(DL_, WM_, WK_, TN_) \
    if (c.dl == DL_ && c.wm == WM_ && c.wk == WK_ && c.tn == TN_) return launch_cfg<T, DL_, WM_, WK_, TN_>(p);
    KS_FMA_CASE(8, 1, 1, 16)
    KS_FMA_CASE(8, 1, 1, 12)
    KS_FMA_CASE(8, 1, 1, 8)
    KS_FMA_CASE(4, 2, 1, 16)
    KS_FMA_CASE(4, 2, 1, 12)
    KS_FMA_CASE(4, 1, 2, 16)
    KS_FMA_CASE(4, 1, 2, 12)
    KS_FMA_CASE(2, 2, 2, 16)
    KS_FMA_CASE(2, 2, 2, 12)
    KS_FMA_CASE(2, 4, 1, 16)
    KS_FMA_CASE(2, 4, 1, 12)
    KS_FMA_CASE(1, 2, 4, 16)
    KS_FMA_CASE(1, 2, 4, 12)
    KS_FMA_CASE(1, 4, 2, 16)
    KS_FMA_CASE(1, 4, 2, 12)
    KS_FMA_CASE(1, 8, 1, 16)
    KS_FMA_CASE(1, 8, 1, 12)
#undef KS_FMA_CASE
    return cudaErrorInvalidConfiguration;
}

}  // namespace

// Tile configurations compiled above, as (dl, wm, wk, tn).
static const FmaConfig kFmaConfigs[] = {
    {8, 1, 1, 16}, {8, 1, 1, 12}, {8, 1, 1, 8},  {4, 2, 1, 16}, {4, 2, 1, 12}, {4, 1, 2, 16},
    {4, 1, 2, 12}, {2, 2, 2, 16}, {2, 2, 2, 12}, {2, 4, 1, 16}, {2, 4, 1, 12}, {1, 2, 4, 16},
    {1, 2, 4, 12}, {1, 4, 2, 16}, {1, 4, 2, 12}, {1, 8, 1, 16}, {1, 8, 1, 12},
};

// l values per CTA for this d, or 0 if the vector loaders cannot serve it.
static int fma_dl(const Problem &p) {
    const int E = p.dtype == KS_BF16 ? 8 : 4;
    if (p.d % 8 == 0) return (8 % E == 0) ? 8 : 0;
    if (p.d == 4 || p.d == 2 || p.d == 1) return (int)p.d;
    if (p.d % 4 == 0 && E == 4) return 4;
    return 0;
}

bool fma_supported(const Problem &p, const char **why) {
    const int E = p.dtype == KS_BF16 ? 8 : 4;
    const int dl = fma_dl(p);
    if (!dl) { *why = "d not served by the vector loaders"; return false; }
    const uintptr_t al = reinterpret_cast<uintptr_t>(p.X) | reinterpret_cast<uintptr_t>(p.V) |
                         reinterpret_cast<uintptr_t>(p.Y);
    if (al % 16) { *why = "X, values and Y must be 16-byte aligned"; return false; }
    if (p.c % E) { *why = "c must be a multiple of the 16-byte element count"; return false; }
    if (dl < E) {
        // runs of JT*d contiguous elements: a 16-byte unit must not cross the
        // end of the block, in X (c*d) or in Y (b*d)
        if ((p.c * p.d) % E || (p.b * p.d) % E) { *why = "c*d and b*d must be multiples of the 16-byte element count"; return false; }
        if ((kJT * dl) % E) { *why = "stage width"; return false; }
    }
    return true;
}

FmaConfig fma_choose(const Problem &p) {
    const int dl = fma_dl(p);
    FmaConfig best = {0, 0, 0, 0};
    double best_score = -1.0;
    for (const FmaConfig &c : kFmaConfigs) {
        if (c.dl != dl) continue;
        const int bm = 64 * c.wm, bkl = 4 * c.tn * c.wk;
        const double kb = (double)((p.b + bkl - 1) / bkl);
        const double waste_k = kb * bkl / (double)p.b;          // >= 1
        const double rb = (double)((p.batch + bm - 1) / bm);
        const double waste_n = rb * bm / (double)p.batch;       // >= 1
        const double reuse = (double)bm * bkl / (bm + bkl);     // FMAs per staged element
        // tiles per wave: fewer tiles than SMs leaves SMs idle
        const double tiles = rb * kb * (double)(p.a * (p.d / dl));
        const double sms = 148.0;
        const double fill = std::min(1.0, tiles / sms);
        const double score = reuse * fill / (waste_k * waste_n);
        if (score > best_score) { best_score = score; best = c; }
    }
    return best;
}

cudaError_t launch_fma(const Problem &p, const FmaConfig &c) {
    if (p.dtype == KS_BF16) return launch_typed<__nv_bfloat16>(p, c);
    // fp32 (KS_F32, and KS_TF32 computed in full fp32) runs on the cp.async
    // ring kernel; this register-staged one remains for grids whose tile count
    // does not fit its 32-bit tile index.
    const cudaError_t e = launch_fma32(p, c);
    if (e != cudaErrorInvalidConfiguration) return e;
    return launch_typed<float>(p, c);
}

}  // namespace ks
