// Output-stationary CUDA-core gather-GEMM for fp32 KS products, with a
// cp.async shared-memory ring.
//
// Y[n, i*b*d + k*d + l] = sum_{j<c} values[i, l, k, j] * X[n, i*c*d + j*d + l]
// (taxoreview.com page on Kronecker-sparse matrix multiplication, first
// abstract: a fused, output-stationary kernel with no permutation passes).
//
// The tile is the one of ks_fma.cu: BM = 64*WM rows x BKL = 4*TN*WK values of
// k x DL consecutive l for one block i, accumulated in registers over all j;
// each warp owns one l and a 64 x (4*TN) piece, each thread 8 rows x TN
// values of k.  Operands reach shared memory without passing through
// registers, in a ring of 3 stages (4 for DL = 4) of 8 j per stage whose
// copies run ahead of the compute, across tile boundaries too:
//
//   X       16-byte cp.async of whole row segments, kept in X's own order:
//           As[n][j*DL + l] (row stride RA = 8*DL + 4 words, RA/4 odd);
//   values  4-byte cp.async into Bs[l][j][k] (k contiguous), lanes = 8 j x 4 k
//           so every copy warp-instruction hits 32 distinct banks.
//
// A thread's rows are interleaved (lane_r + 8 m), so its 8 scalar loads of A
// per j hit 8 distinct banks; its k are 4 consecutive per 16, read as float4.
// Products use fma.rn.f32x2, on pairs of k (DL == 1) or pairs of rows.
//
// Rounding: every product and sum is an fp32 fma.rn, j = 0..c-1 per output.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdint>

#include "ks_epilogue.cuh"
#include "ks_internal.h"

namespace ks {
namespace {

constexpr int kThreads = 256;
constexpr int kJT = 8;   // j per stage

struct Fma32Params {
    const float *X;
    const float *V;
    float *Y;
    const float *bias;  // fused epilogue: out_f values or null
    int act;
    long long N;
    int a, b, c, d;
    int bc;  // b * c
    int in_f, out_f;
    int n_g, n_kb, n_stages;
    int n_tiles;
};

template <int DL, int WM, int WK, int TN>
struct Tile32 {
    static_assert(DL * WM * WK == 8, "8 warps per CTA");
    static constexpr int BM = 64 * WM;
    static constexpr int BKL = 4 * TN * WK;
    static constexpr int RA = kJT * DL + 4;           // As row stride (words), RA/4 odd
    static constexpr int A_WORDS = BM * RA;
    static constexpr int BKP = BKL + 4;               // Bs j-row stride, = 4 (mod 32) or 20
    static constexpr int PSB = kJT * BKP + 4;         // Bs plane stride
    static constexpr int STAGE = A_WORDS + DL * PSB;  // words
    static constexpr int RS = DL * BKP + (DL == 1 ? 0 : 4);  // epilogue row stride, = 4 (mod 8)
    // the epilogue stages all rows at once if that fits beside the ring, else
    // half of each warp's 64 rows per pass
    // ring depth: 3 stages; 4 for DL = 4, the one l width a fourth stage made
    // faster (elsewhere it was slower: the larger shared-memory carve-out
    // leaves less L1 for the 4-byte values copies)
    static constexpr int NS = (DL == 4 && (4 * STAGE + BM / 2 * RS) * 4 <= 232448) ? 4 : 3;
    static constexpr int NP = (NS * STAGE + BM * RS) * 4 <= 232448 ? 1 : 2;
    static constexpr int EPI = BM / NP * RS;
    static constexpr int SMEM_FLOATS = NS * STAGE + EPI;
    static constexpr int CA = 2 * DL;                 // 16-byte chunks per A row per stage
    static constexpr int NXC = (BM * CA + kThreads - 1) / kThreads;      // A copies per thread
    static constexpr int NV = (DL * BKL * kJT + kThreads - 1) / kThreads;  // values copies per thread
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const float *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const float *src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async16_full(uint32_t dst, const float *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4_full(uint32_t dst, const float *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// VT: p.V holds the values transposed per block, vt[i][l][j][k] (k
// contiguous), and goes to shared memory with 16-byte copies; otherwise the
// values keep their [i][l][k][j] layout and move as 4-byte transposing copies.
template <int DL, int WM, int WK, int TN, bool VT>
__global__ void __launch_bounds__(kThreads, 1) fma32_kernel(const Fma32Params p) {
    using TL = Tile32<DL, WM, WK, TN>;
    constexpr int BM = TL::BM, BKL = TL::BKL;
    extern __shared__ __align__(16) float smem[];
    constexpr int kNS = TL::NS;
    float *sEpi = smem + kNS * TL::STAGE;
    const uint32_t s_base = (uint32_t)__cvta_generic_to_shared(smem);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int w_l = warp / (WM * WK);
    const int w_m = (warp / WK) % WM;
    const int w_k = warp % WK;
    const int lane_r = lane >> 2, lane_k = lane & 3;
    const int groups_per_i = p.d / DL;
    const int S = p.n_stages;
    const int my_tiles = (p.n_tiles > (int)blockIdx.x) ? (p.n_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

    // Per-thread copy roles, fixed for the whole kernel.
    //   X: chunk q = tid % CA of rows tid / CA + t * XR (t < NXC): elements
    //      f = 4q..4q+3 of the row's (j * DL + l), i.e. j = jx, l = lx..lx+3.
    //   values: j = vj, k = kq + (32 t) % BKL, l = (32 t) / BKL (t < NV).
    constexpr int XR = kThreads / TL::CA;
    const int xn = tid / TL::CA, xf = 4 * (tid % TL::CA);
    const int jx = xf / DL, lx = xf % DL;
    const int vj = lane & 7, kq = tid >> 3;
    const long long x_row_step = (long long)XR * p.in_f;
    // VT copies: element e = tid + 256 t of the stage's (l, j, 4-k group), k fastest
    constexpr int K4 = BKL / 4, NVT = (DL * kJT * K4 + kThreads - 1) / kThreads;

    // Copy state: the next stage to issue is stage iss_s of tile iteration iss_it.
    int iss_it = 0, iss_s = 0, iss_buf = 0;
    const float *x_thr = p.X;  // this thread's first X chunk of the tile, at j = 0
    const float *v_thr = p.V;  // values[i][l0][k0 + kq][vj] (VT: vt[i][l0][0][k0])
    int x_rows = 0;            // rows left from this thread's first copy row
    int k_left = 0;            // p.b - k0 - kq
    bool full = false;         // every row and every k of the tile in range
    auto set_issue_tile = [&](int it) {
        const int tile = (int)blockIdx.x + it * (int)gridDim.x;
        const int kb = tile % p.n_kb;
        const int rest = tile / p.n_kb;
        const int gg = rest % p.n_g;
        const long long n0 = (long long)(rest / p.n_g) * BM;
        const int i = gg / groups_per_i, l0 = (gg % groups_per_i) * DL;
        const int k0 = kb * BKL;
        x_rows = (int)min((long long)(BM + 1), p.N - n0) - xn;
        k_left = p.b - k0 - kq;
        full = (n0 + BM <= p.N) && (k0 + BKL <= p.b);
        x_thr = p.X + (n0 + xn) * p.in_f + (long long)i * p.c * p.d + (long long)jx * p.d + l0 + lx;
        if constexpr (VT)
            v_thr = p.V + (long long)(i * p.d + l0) * p.c * p.b + k0;
        else
            v_thr = p.V + ((long long)(i * p.d + l0) * p.b + k0 + kq) * p.c + vj;
    };
    if (my_tiles > 0) set_issue_tile(0);

    // values copy t: l = lt(t), k = kq + kt(t); its source offset from v_thr
    auto v_lk = [&](int t, int &l, int &kc) {
        if constexpr (BKL % 32 == 0) {
            kc = (32 * t) % BKL;
            l = (32 * t) / BKL;
        } else {  // e = kq + 32 t split at runtime (BKL not a multiple of 32)
            const int e8 = kq + 32 * t;
            l = e8 / BKL;
            kc = e8 % BKL - kq;
        }
    };

    // Issues the copies of the next stage (if any is left) and commits a group.
    auto issue = [&]() {
        if (iss_it < my_tiles) {
            const int j0 = iss_s * kJT;
            const uint32_t st = s_base + (uint32_t)(iss_buf * TL::STAGE) * 4u;
            const uint32_t sx = st + (uint32_t)(xn * TL::RA + xf) * 4u;
            const uint32_t sv = st + (uint32_t)(TL::A_WORDS + vj * TL::BKP + kq) * 4u;
            const float *xs = x_thr + (long long)j0 * p.d;
            const float *vs = v_thr + j0;
            if (full && j0 + kJT <= p.c) {
#pragma unroll
                for (int t = 0; t < TL::NXC; ++t)
                    if (TL::NXC * kThreads == BM * TL::CA || xn + t * XR < BM)
                        cp_async16_full(sx + (uint32_t)(t * XR * TL::RA) * 4u, xs + t * x_row_step);
                if constexpr (VT) {
#pragma unroll
                    for (int t = 0; t < NVT; ++t) {
                        const int e = tid + t * kThreads;
                        if (NVT * kThreads == DL * kJT * K4 || e < DL * kJT * K4) {
                            const int k4 = e % K4, jl = e / K4, j = jl % kJT, l = jl / kJT;
                            cp_async16_full(st + (uint32_t)(TL::A_WORDS + l * TL::PSB + j * TL::BKP + 4 * k4) * 4u,
                                            v_thr + ((long long)(l * p.c + j0 + j) * p.b + 4 * k4));
                        }
                    }
                } else {
#pragma unroll
                    for (int t = 0; t < TL::NV; ++t) {
                        int l, kc;
                        v_lk(t, l, kc);
                        if (BKL % 32 == 0 || TL::NV * kThreads == DL * BKL * kJT || kq + 32 * t < DL * BKL)
                            cp_async4_full(sv + (uint32_t)(l * TL::PSB + kc) * 4u, vs + (l * p.bc + kc * p.c));
                    }
                }
            } else {
                const bool jxv = j0 + jx < p.c;
#pragma unroll
                for (int t = 0; t < TL::NXC; ++t) {
                    if (TL::NXC * kThreads == BM * TL::CA || xn + t * XR < BM) {
                        const bool v = jxv && t * XR < x_rows;
                        cp_async16(sx + (uint32_t)(t * XR * TL::RA) * 4u, v ? xs + t * x_row_step : p.X, v);
                    }
                }
                if constexpr (VT) {
#pragma unroll
                    for (int t = 0; t < NVT; ++t) {
                        const int e = tid + t * kThreads;
                        if (NVT * kThreads == DL * kJT * K4 || e < DL * kJT * K4) {
                            const int k4 = e % K4, jl = e / K4, j = jl % kJT, l = jl / kJT;
                            const bool v = (j0 + j < p.c) && (4 * k4 < k_left + kq);  // k_left + kq = b - k0
                            cp_async16(st + (uint32_t)(TL::A_WORDS + l * TL::PSB + j * TL::BKP + 4 * k4) * 4u,
                                       v ? v_thr + ((long long)(l * p.c + j0 + j) * p.b + 4 * k4) : p.V, v);
                        }
                    }
                } else {
                    const bool jvv = j0 + vj < p.c;
#pragma unroll
                    for (int t = 0; t < TL::NV; ++t) {
                        int l, kc;
                        v_lk(t, l, kc);
                        if (BKL % 32 == 0 || TL::NV * kThreads == DL * BKL * kJT || kq + 32 * t < DL * BKL) {
                            const bool v = jvv && kc < k_left;
                            cp_async4(sv + (uint32_t)(l * TL::PSB + kc) * 4u, v ? vs + (l * p.bc + kc * p.c) : p.V, v);
                        }
                    }
                }
            }
            if (++iss_s == S) {
                iss_s = 0;
                if (++iss_it < my_tiles) set_issue_tile(iss_it);
            }
        }
        iss_buf = (iss_buf + 1 == kNS) ? 0 : iss_buf + 1;
        cp_async_commit();  // one group per stage, empty or not
    };

#pragma unroll
    for (int g = 0; g < kNS - 1; ++g) issue();

    // Accumulator pairs for fma.rn.f32x2.  DL == 1: acc[m][2q + h] holds row
    // a_row + 8m at k = b_col + 16q + 2h + (0, 1), X broadcast over a k pair.
    // DL > 1: acc[pr][kk] holds rows a_row + 16pr + (0, 8) at the thread's
    // kk-th k (b_col + 16(kk/4) + kk%4), the weight broadcast over a row pair.
    // (Both are 4 x 2 TN fp32 sums; which one runs faster depends on DL.)
    constexpr bool kPairK = (DL == 1);
    float2 acc[8][TN / 2];
    int buf = 0;  // ring buffer of the stage being computed
    const int a_row = w_m * 64 + lane_r;                        // thread rows a_row + 8 m
    const int b_col = w_k * (4 * TN) + lane_k * 4;               // thread k: b_col + 16 q + e
    for (int it = 0; it < my_tiles; ++it) {
        const int tile = (int)blockIdx.x + it * (int)gridDim.x;
#pragma unroll
        for (int m = 0; m < 8; ++m)
#pragma unroll
            for (int kk = 0; kk < TN / 2; ++kk) acc[m][kk] = make_float2(0.f, 0.f);

        for (int s = 0; s < S; ++s) {
            cp_async_wait<kNS - 2>();
            __syncthreads();
            issue();  // into the buffer computed one step ago
            const float *stage = smem + buf * TL::STAGE;
            buf = (buf + 1 == kNS) ? 0 : buf + 1;
            const float *As = stage + a_row * TL::RA + w_l;
            const float *Bs = stage + TL::A_WORDS + w_l * TL::PSB + b_col;
#pragma unroll
            for (int jj = 0; jj < kJT; ++jj) {
                float am[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) am[m] = As[m * 8 * TL::RA + jj * DL];
                float4 bq[TN / 4];
#pragma unroll
                for (int q = 0; q < TN / 4; ++q) bq[q] = *reinterpret_cast<const float4 *>(Bs + jj * TL::BKP + 16 * q);
                if constexpr (kPairK) {
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const float2 a2 = make_float2(am[m], am[m]);
#pragma unroll
                        for (int q = 0; q < TN / 4; ++q) {
                            acc[m][2 * q] = __ffma2_rn(a2, make_float2(bq[q].x, bq[q].y), acc[m][2 * q]);
                            acc[m][2 * q + 1] = __ffma2_rn(a2, make_float2(bq[q].z, bq[q].w), acc[m][2 * q + 1]);
                        }
                    }
                } else {
                    // acc viewed as [4][TN]: acc[pr][kk] at flat index pr * TN + kk
                    float2 *ac = &acc[0][0];
#pragma unroll
                    for (int pr = 0; pr < 4; ++pr) {
                        const float2 ap = make_float2(am[2 * pr], am[2 * pr + 1]);
#pragma unroll
                        for (int q = 0; q < TN / 4; ++q) {
                            float2 *r = ac + pr * TN + 4 * q;
                            r[0] = __ffma2_rn(ap, make_float2(bq[q].x, bq[q].x), r[0]);
                            r[1] = __ffma2_rn(ap, make_float2(bq[q].y, bq[q].y), r[1]);
                            r[2] = __ffma2_rn(ap, make_float2(bq[q].z, bq[q].z), r[2]);
                            r[3] = __ffma2_rn(ap, make_float2(bq[q].w, bq[q].w), r[3]);
                        }
                    }
                }
            }
        }

        // Epilogue through its own shared region (the next tile's first stages
        // are already in flight): Cs[row][l][k], then 16-byte stores of Y.
        const int kb = tile % p.n_kb;
        const int rest = tile / p.n_kb;
        const int gg = rest % p.n_g;
        const long long n0 = (long long)(rest / p.n_g) * BM;
        const int i = gg / groups_per_i, l0 = (gg % groups_per_i) * DL;
        const int k0 = kb * BKL;
        constexpr int NP = TL::NP, MP = 8 / NP, RW = 64 / NP;  // rows per warp and pass
#pragma unroll
        for (int h = 0; h < NP; ++h) {
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) {
                const int m = h * MP + mm;
                float *dst = sEpi + (w_m * RW + lane_r + 8 * mm) * TL::RS + w_l * TL::BKP + b_col;
#pragma unroll
                for (int q = 0; q < TN / 4; ++q) {
                    float4 o;
                    if constexpr (kPairK) {
                        o = make_float4(acc[m][2 * q].x, acc[m][2 * q].y, acc[m][2 * q + 1].x, acc[m][2 * q + 1].y);
                    } else {
                        const float2 *r = &acc[0][0] + (m / 2) * TN + 4 * q;
                        o = (m % 2 == 0) ? make_float4(r[0].x, r[1].x, r[2].x, r[3].x)
                                         : make_float4(r[0].y, r[1].y, r[2].y, r[3].y);
                    }
                    *reinterpret_cast<float4 *>(dst + 16 * q) = o;
                }
            }
            __syncthreads();
            constexpr int UO = BKL * DL / 4;  // 16-byte output units per row
            for (int idx = tid; idx < BM / NP * UO; idx += kThreads) {
                const int rr = idx / UO;
                const int uo = idx - rr * UO;
                const long long row = n0 + (rr / RW) * 64 + h * RW + rr % RW;
                const int f = uo * 4;  // flat (k_local, l_local)
                const int kl = f / DL, ll = f % DL;
                if (row < p.N && k0 + kl < p.b) {
                    float v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int fe = f + e;
                        v[e] = sEpi[rr * TL::RS + (fe % DL) * TL::BKP + fe / DL];
                    }
                    const long long col = (long long)i * p.b * p.d + (long long)(k0 + kl) * p.d + l0 + ll;
                    if (p.bias) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) v[e] += ep_bias(p.bias, col + e);
                    }
                    if (p.act) ep_act_array(v, p.act);
                    *reinterpret_cast<float4 *>(p.Y + row * p.out_f + col) = make_float4(v[0], v[1], v[2], v[3]);
                }
            }
            __syncthreads();
        }
    }
    cp_async_wait<0>();  // no copy may still be landing when the CTA exits
}

template <int DL, int WM, int WK, int TN>
cudaError_t launch_cfg32(const Problem &pr, const float *vt) {
    using TL = Tile32<DL, WM, WK, TN>;
    Fma32Params p;
    p.X = static_cast<const float *>(pr.X);
    p.V = vt ? vt : static_cast<const float *>(pr.V);
    p.Y = static_cast<float *>(pr.Y);
    p.bias = static_cast<const float *>(pr.bias);
    p.act = pr.act;
    p.N = pr.batch;
    p.a = (int)pr.a; p.b = (int)pr.b; p.c = (int)pr.c; p.d = (int)pr.d;
    p.bc = (int)(pr.b * pr.c);
    p.in_f = (int)pr.in_features();
    p.out_f = (int)pr.out_features();
    p.n_g = (int)(pr.a * (pr.d / DL));
    p.n_kb = (int)((pr.b + TL::BKL - 1) / TL::BKL);
    p.n_stages = (int)((pr.c + kJT - 1) / kJT);
    const long long n_rb = (pr.batch + TL::BM - 1) / TL::BM;
    const long long n_tiles = n_rb * p.n_g * p.n_kb;
    if (n_tiles > INT32_MAX - 4096) return cudaErrorInvalidConfiguration;  // tile indices are 32-bit
    p.n_tiles = (int)n_tiles;
    const size_t smem = (size_t)TL::SMEM_FLOATS * sizeof(float);
    if (smem > 232448) return cudaErrorInvalidConfiguration;
    auto kern = vt ? fma32_kernel<DL, WM, WK, TN, true> : fma32_kernel<DL, WM, WK, TN, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = std::min<long long>(p.n_tiles, (long long)sm_count());
    kern<<<(int)grid, kThreads, smem, pr.stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

namespace {

cudaError_t launch_cfg_any(const Problem &p, const FmaConfig &c, const float *vt) {
#define KS_FMA32_CASE(DL_, WM_, WK_, TN_) \
    if (c.dl == DL_ && c.wm == WM_ && c.wk == WK_ && c.tn == TN_) return launch_cfg32<DL_, WM_, WK_, TN_>(p, vt);
    KS_FMA32_CASE(8, 1, 1, 16)
    KS_FMA32_CASE(8, 1, 1, 12)
    KS_FMA32_CASE(8, 1, 1, 8)
    KS_FMA32_CASE(4, 2, 1, 16)
    KS_FMA32_CASE(4, 2, 1, 12)
    KS_FMA32_CASE(4, 1, 2, 16)
    KS_FMA32_CASE(4, 1, 2, 12)
    KS_FMA32_CASE(2, 2, 2, 16)
    KS_FMA32_CASE(2, 2, 2, 12)
    KS_FMA32_CASE(2, 4, 1, 16)
    KS_FMA32_CASE(2, 4, 1, 12)
    KS_FMA32_CASE(1, 2, 4, 16)
    KS_FMA32_CASE(1, 2, 4, 12)
    KS_FMA32_CASE(1, 4, 2, 16)
    KS_FMA32_CASE(1, 4, 2, 12)
    KS_FMA32_CASE(1, 8, 1, 16)
    KS_FMA32_CASE(1, 8, 1, 12)
#undef KS_FMA32_CASE
    return cudaErrorInvalidConfiguration;
}

}  // namespace

// With 8 l per tile (d % 8 == 0), products large enough to amortise it
// (>= 2^30 flop, values <= 64 MiB, b % 4 == 0) first transpose the values per
// block into a workspace from the library's pool, so the kernel stages them
// with 16-byte copies instead of four times as many 4-byte ones; the
// workspace is freed on the stream after the kernel.  Measured against the
// in-place path on the fp32 sweep: 1.20x median for d % 8 == 0; for smaller
// l widths the gain (1.01-1.03x) did not cover the transpose on mid-size runs.
// If the workspace cannot be had, the values are read in place.
cudaError_t launch_fma32(const Problem &p, const FmaConfig &c) {
    const long long nvals = p.a * p.b * p.c * p.d;
    const double flops = 2.0 * (double)p.batch * (double)nvals;
    if (c.dl == 8 && p.b % 4 == 0 && flops >= 1073741824.0 && nvals * 4 <= (64LL << 20)) {
        cudaMemPool_t pool = chain_pool();
        void *vt = nullptr;
        if (pool && cudaMallocFromPoolAsync(&vt, (size_t)nvals * 4, pool, p.stream) == cudaSuccess) {
            cudaError_t e = launch_transpose_blocks(p.V, vt, p.a * p.d, p.b, p.c, KS_F32, p.stream);
            if (e == cudaSuccess) e = launch_cfg_any(p, c, static_cast<const float *>(vt));
            const cudaError_t ef = cudaFreeAsync(vt, p.stream);
            return e != cudaSuccess ? e : ef;
        }
        (void)cudaGetLastError();
    }
    return launch_cfg_any(p, c, nullptr);
}

}  // namespace ks
