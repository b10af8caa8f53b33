// Output-stationary CUDA-core gather-GEMM for fp32 KS products, with a
// cp.async shared-memory ring.
//
// Y[n, i*b*d + k*d + l] = sum_{j<c} values[i, l, k, j] * X[n, i*c*d + j*d + l]
// (taxoreview.com page on Kronecker-sparse matrix multiplication, first
// abstract: a fused, output-stationary kernel with no permutation passes).
//
// A tile is BM rows x BKL values of k x DL consecutive l of one block i,
// accumulated in registers over all j.  Every warp spans all DL l of its
// tile: its 32 lanes are RG row groups x DL values of l x KQ groups of k
// (KQ = 1, 1, 2, 4 and RG = 4, 8, 8, 8 for DL = 8, 4, 2, 1), and a thread owns
// 8 rows (rg + RG*m) x TN values of k (4 consecutive per group) of one l.  The
// outputs Y[n][k*d + l0 .. l0+DL-1] of a row and k thus sit in neighbouring
// lanes and leave straight from registers: no shared-memory interleave of
// the l, no barrier after a tile.  Operands reach shared memory without passing
// through registers, in a ring of stages of 8 j whose copies run ahead of the
// compute, across tile boundaries too.  A warpgroup of its own (warps 8-11)
// issues the copies; the eight compute warps (0-7) meet it only at each
// stage's full and empty mbarriers:
//
//   X       16-byte cp.async of whole row segments, kept in X's own order:
//           As[n][j*DL + l], row stride RA chosen so that one warp's loads
//           (RG rows x DL l) fall in distinct banks;
//   values  4-byte cp.async into Bs[l][j][k] (k contiguous), lanes = 8 j x 4 k
//           so every copy warp-instruction hits 32 distinct banks; or, from a
//           per-call transposed copy, 16-byte copies.  The l planes are PSB
//           words apart so that one warp's DL (x KQ) 16-byte loads are distinct.
//
// Products use fma.rn.f32x2 on pairs of k, the X value broadcast.
//
// Rounding: every product and sum is an fp32 fma.rn, j = 0..c-1 per output.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <type_traits>

#include "ks_epilogue.cuh"
#include "ks_internal.h"
#include "ks_sm100.cuh"

namespace ks {
namespace {

constexpr int kThreads = 384;    // eight compute warps, then a copy-issuing warpgroup
constexpr int kCopyRoles = 256;  // copy roles per stage (two per copy thread)
constexpr int kJT = 8;           // j per stage

struct Fma32Params {
    unsigned *status;
    const float *X;
    const float *V;
    float *Y;
    const float *bias;  // fused epilogue: out_f values or null
    int bias_vec4;      // bias is 16-byte aligned: read four columns at once
    int act;
    long long N;
    int a, b, c, d;
    int bc;  // b * c
    int in_f, out_f;
    int n_g, n_kb, n_stages;
    int n_tiles;
};

// Lane geometry per l width: KQ lane groups along k, RG along rows; RA is the
// As row stride (words): RA*rg + l over a warp's RG x DL loads hits 32
// distinct banks (or 16 distinct pairs for DL = 2), and rows stay 16-byte
// aligned for the copies.
template <int DL>
struct Lanes32 {
    static constexpr int KQ = DL == 2 ? 2 : DL == 1 ? 4 : 1;
    static constexpr int RG = 32 / (DL * KQ);
    static constexpr int RA = DL == 8 ? 72 : DL == 4 ? 36 : DL == 2 ? 20 : 12;
};

template <int DL, int WM, int WK, int TN>
struct Tile32 {
    using LN = Lanes32<DL>;
    static_assert(WM * WK == 8, "8 warps per CTA");
    static_assert(TN % 4 == 0, "k per thread in groups of 4");
    static constexpr int BM = 8 * LN::RG * WM;        // rows per tile (a warp: 8 row groups)
    static constexpr int KW = LN::KQ * TN;            // k per warp
    static constexpr int BKL = KW * WK;               // k per tile
    static constexpr int RA = LN::RA;
    static constexpr int A_WORDS = BM * RA;
    static constexpr int BKP = BKL + 4;               // Bs j-row stride, = 4 (mod 32) or 20
    // plane stride: PSB/4 odd (DL = 8, 4) or = 2 (mod 8) (DL = 2, with the k pair of lanes)
    static constexpr int PSB = kJT * BKP + (DL == 2 ? 8 : 4);
    static constexpr int STAGE = A_WORDS + DL * PSB;  // words
    // ring depth: 4 stages for DL = 4, 3 otherwise (measured: a fourth stage
    // helps DL = 4; for the other widths the larger shared-memory carve-out
    // leaves less L1 for the 4-byte values copies, 1-2% slower)
    static constexpr int NS = (DL == 4 && 4 * STAGE * 4 <= 232448) ? 4 : 3;
    static constexpr int SMEM_FLOATS = NS * STAGE;
    static constexpr int CA = 2 * DL;                 // 16-byte chunks per A row per stage
    static constexpr int NXC = (BM * CA + kCopyRoles - 1) / kCopyRoles;  // A copies per role
};

// Activation ACT (0 none, 1 ReLU, 2 GELU tanh form, 3 GELU erf form) of four
// outputs, chosen at compile time.
template <int ACT>
__device__ __forceinline__ void ep_act4(float (&v)[4]) {
    if constexpr (ACT == 2) {  // in pairs (ViT bias + GELU: 1.23x against the earlier scalar tanh form)
        const float2 a = gelu_tanh_f2(make_float2(v[0], v[1]));
        const float2 b = gelu_tanh_f2(make_float2(v[2], v[3]));
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
        return;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        if constexpr (ACT == 1) v[e] = fmaxf(v[e], 0.f);
        if constexpr (ACT == 3) v[e] = gelu_erf_f(v[e]);
    }
}

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
// The mbarrier receives one arrival when every cp.async this thread issued
// before it has landed (.noinc: that arrival is one of the barrier's expected
// count).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(sm100::su32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// VT: p.V holds the values transposed per block, vt[i][l][j][k] (k
// contiguous), and goes to shared memory with 16-byte copies; otherwise the
// values keep their [i][l][k][j] layout and move as 4-byte transposing copies.
//
// Warps 8-11 issue every copy: each of their 128 threads plays two of the
// stage's 256 copy roles and signals the stage's full barrier when its copies
// have landed (cp.async.mbarrier.arrive.noinc, 128 arrivals per phase).  Warps
// 0-7 only compute: they wait for full stages and release them through the
// empty barriers (one arrival per warp), so warps drift apart and one warp's
// epilogue overlaps the others' products; no CTA-wide barrier runs after the
// start.  The copy warpgroup gives registers to the compute warps
// (setmaxnreg: 128 x 40 + 256 x 232 = the 384 x 168 of the launch).  Every
// wait is bounded; a wait that runs out sets the device status word and the
// CTA's abort flag, which ends every role's loop.
template <int DL, int WM, int WK, int TN, bool VT>
__global__ void __launch_bounds__(kThreads, 1) fma32_kernel(const Fma32Params p) {
    using TL = Tile32<DL, WM, WK, TN>;
    constexpr int BM = TL::BM, BKL = TL::BKL;
    using LN = typename TL::LN;
    extern __shared__ __align__(16) float smem[];
    constexpr int kNS = TL::NS;
    constexpr int kBarOff = (TL::SMEM_FLOATS * 4 + 15) / 16 * 16;  // bytes
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(smem) + kBarOff);
    uint64_t *empty_bar = full_bar + kNS;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty_bar + kNS);
    const uint32_t s_base = (uint32_t)__cvta_generic_to_shared(smem);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int groups_per_i = p.d / DL;
    const int S = p.n_stages;
    const int my_tiles = (p.n_tiles > (int)blockIdx.x) ? (p.n_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

    if (tid == 0) {
        for (int s = 0; s < kNS; ++s) {
            sm100::mbar_init(&full_bar[s], 128);
            sm100::mbar_init(&empty_bar[s], 8);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp >= 8) {
        // ------------------------------------------------ copy issue (warps 8-11, two copy roles per thread)
        // registers: 256 x 232 + 128 x 40 = 64512 = 384 threads x 168 at launch
        asm volatile("setmaxnreg.dec.sync.aligned.u32 40;" ::: "memory");
        const int pt = threadIdx.x - 256;  // 0..127
        constexpr int kT = kCopyRoles;
        constexpr int XR = kT / TL::CA;
        constexpr int K4 = BKL / 4, NVT = (DL * kJT * K4 + kT - 1) / kT;
        constexpr int NV = (DL * BKL * kJT + kT - 1) / kT;
        const long long x_row_step = (long long)XR * p.in_f;
        uint32_t fill = 0;
        bool ok = true;
        for (int it = 0; it < my_tiles && ok; ++it) {
            const int tile = (int)blockIdx.x + it * (int)gridDim.x;
            const int kb = tile % p.n_kb;
            const int rest = tile / p.n_kb;
            const int gg = rest % p.n_g;
            const long long n0 = (long long)(rest / p.n_g) * BM;
            const int i = gg / groups_per_i, l0 = (gg % groups_per_i) * DL;
            const int k0 = kb * BKL;
            const bool full_t = (n0 + BM <= p.N) && (k0 + BKL <= p.b);
            for (int s = 0; s < S && ok; ++s, ++fill) {
                const int buf = (int)(fill % kNS);
                ok = sm100::mbar_wait(&empty_bar[buf], ((fill / kNS) & 1) ^ 1, abort_flag, p.status);
                if (!ok) break;
                const int j0 = s * kJT;
                const uint32_t st = s_base + (uint32_t)(buf * TL::STAGE) * 4u;
                const bool fast = full_t && j0 + kJT <= p.c;
#pragma unroll 1
                for (int v = 0; v < kT / (kThreads - 256); ++v) {
                    const int vt = pt + 128 * v;
                    const int xn = vt / TL::CA, xf = 4 * (vt % TL::CA);
                    const int jx = xf / DL, lx = xf % DL;
                    const int vj = vt & 7, kq = vt >> 3;
                    const float *xs = p.X + (n0 + xn) * p.in_f + (long long)i * p.c * p.d + (long long)(j0 + jx) * p.d +
                                      l0 + lx;
                    const uint32_t sx = st + (uint32_t)(xn * TL::RA + xf) * 4u;
                    const int x_rows = (int)min((long long)(BM + 1), p.N - n0) - xn;
                    const bool jxv = j0 + jx < p.c;
#pragma unroll
                    for (int t = 0; t < TL::NXC; ++t) {
                        if (TL::NXC * kT == BM * TL::CA || xn + t * XR < BM) {
                            if (fast) {
                                cp_async16_full(sx + (uint32_t)(t * XR * TL::RA) * 4u, xs + t * x_row_step);
                            } else {
                                const bool ok2 = jxv && t * XR < x_rows;
                                cp_async16(sx + (uint32_t)(t * XR * TL::RA) * 4u, ok2 ? xs + t * x_row_step : p.X, ok2);
                            }
                        }
                    }
                    if constexpr (VT) {
                        const float *vbase = p.V + (long long)(i * p.d + l0) * p.c * p.b + k0;
#pragma unroll
                        for (int t = 0; t < NVT; ++t) {
                            const int e = vt + t * kT;
                            if (NVT * kT == DL * kJT * K4 || e < DL * kJT * K4) {
                                const int k4 = e % K4, jl = e / K4, j = jl % kJT, l = jl / kJT;
                                const uint32_t dst = st + (uint32_t)(TL::A_WORDS + l * TL::PSB + j * TL::BKP + 4 * k4) * 4u;
                                const float *src = vbase + ((long long)(l * p.c + j0 + j) * p.b + 4 * k4);
                                if (fast) {
                                    cp_async16_full(dst, src);
                                } else {
                                    const bool ok2 = (j0 + j < p.c) && (4 * k4 < p.b - k0);
                                    cp_async16(dst, ok2 ? src : p.V, ok2);
                                }
                            }
                        }
                    } else {
                        const float *vs = p.V + ((long long)(i * p.d + l0) * p.b + k0 + kq) * p.c + vj + j0;
                        const uint32_t sv = st + (uint32_t)(TL::A_WORDS + vj * TL::BKP + kq) * 4u;
                        const int k_left = p.b - k0 - kq;
                        const bool jvv = j0 + vj < p.c;
#pragma unroll
                        for (int t = 0; t < NV; ++t) {
                            int l, kc;
                            if constexpr (BKL % 32 == 0) {
                                kc = (32 * t) % BKL;
                                l = (32 * t) / BKL;
                            } else {
                                const int e8 = kq + 32 * t;
                                l = e8 / BKL;
                                kc = e8 % BKL - kq;
                            }
                            if (BKL % 32 == 0 || NV * kT == DL * BKL * kJT || kq + 32 * t < DL * BKL) {
                                if (fast) {
                                    cp_async4_full(sv + (uint32_t)(l * TL::PSB + kc) * 4u, vs + (l * p.bc + kc * p.c));
                                } else {
                                    const bool ok2 = jvv && kc < k_left;
                                    cp_async4(sv + (uint32_t)(l * TL::PSB + kc) * 4u, ok2 ? vs + (l * p.bc + kc * p.c) : p.V,
                                              ok2);
                                }
                            }
                        }
                    }
                }
                cp_async_mbar_arrive_noinc(&full_bar[buf]);  // fires when this lane's copies have landed
            }
        }
        cp_async_wait_all();  // no copy may still be landing when the CTA exits
        return;
    }

    // ------------------------------------------------ compute warps 0-7
    asm volatile("setmaxnreg.inc.sync.aligned.u32 232;" ::: "memory");
    const int w_m = warp / WK;
    const int w_k = warp % WK;
    // compute roles: lane = (row group, l, k group), k group fastest
    const int c_kq = lane % LN::KQ, c_l = (lane / LN::KQ) % DL, c_rg = lane / (LN::KQ * DL);
    // acc[m][2q + h]: row a_row + RG*m, k = b_col + 4*KQ*q + 2h + (0, 1), l = l0 + c_l
    float2 acc[8][TN / 2];
    const int a_row = w_m * (8 * LN::RG) + c_rg;
    const int b_col = w_k * TL::KW + 4 * c_kq;
    uint32_t fill = 0;
    bool ok = true;
    for (int it = 0; it < my_tiles && ok; ++it) {
        const int tile = (int)blockIdx.x + it * (int)gridDim.x;
#pragma unroll
        for (int m = 0; m < 8; ++m)
#pragma unroll
            for (int kk = 0; kk < TN / 2; ++kk) acc[m][kk] = make_float2(0.f, 0.f);

        for (int s = 0; s < S; ++s, ++fill) {
            const int buf = (int)(fill % kNS);
            ok = __all_sync(0xffffffffu, sm100::mbar_wait(&full_bar[buf], (fill / kNS) & 1, abort_flag, p.status));
            if (!ok) break;
            const float *stage = smem + buf * TL::STAGE;
            const float *As = stage + a_row * TL::RA + c_l;
            const float *Bs = stage + TL::A_WORDS + c_l * TL::PSB + b_col;
#pragma unroll
            for (int jj = 0; jj < kJT; ++jj) {
                float am[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) am[m] = As[m * LN::RG * TL::RA + jj * DL];
                float4 bq[TN / 4];
#pragma unroll
                for (int q = 0; q < TN / 4; ++q)
                    bq[q] = *reinterpret_cast<const float4 *>(Bs + jj * TL::BKP + 4 * LN::KQ * q);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float2 a2 = make_float2(am[m], am[m]);
#pragma unroll
                    for (int q = 0; q < TN / 4; ++q) {
                        acc[m][2 * q] = __ffma2_rn(a2, make_float2(bq[q].x, bq[q].y), acc[m][2 * q]);
                        acc[m][2 * q + 1] = __ffma2_rn(a2, make_float2(bq[q].z, bq[q].w), acc[m][2 * q + 1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(&empty_bar[buf]);  // this warp is done with the stage
        }
        if (!ok) break;
        // Epilogue straight from registers.  A thread holds, per row m and k group q,
        // four consecutive k of its one l.  Shuffles among the lanes of a row group
        // turn that into four consecutive outputs of Y (DL >= 4: 4x4 transpose over
        // four l lanes -> (one k, four l); DL = 2: exchange between the two l lanes
        // -> (two k, two l); DL = 1: already four k), which leave as one 16-byte
        // store: no shared-memory interleave, no barrier.  The shuffles run on all
        // lanes; only the stores are predicated.
        const int kb = tile % p.n_kb;
        const int rest = tile / p.n_kb;
        const int gg = rest % p.n_g;
        const long long n0 = (long long)(rest / p.n_g) * BM;
        const int i = gg / groups_per_i, l0 = (gg % groups_per_i) * DL;
        const int kt = kb * BKL + b_col;  // the thread's first k
        // output column of the thread's vector for k group q: k_v(q) * d + l_v
        const int r4 = c_l & 3;
        const int l_v = DL >= 4 ? l0 + (c_l & ~3) : l0;
        const int k_off = DL >= 4 ? r4 : DL == 2 ? 2 * c_l : 0;
        const long long colbase = (long long)i * p.b * p.d + l_v;
        // The unrolled store loop, once per activation: the plain copy carries no
        // epilogue code at all; the fused ones add the bias (read once per tile:
        // the thread's TN/4 vectors of columns are the same for its 8 rows) and
        // apply the activation inline.
        auto store_tile = [&](auto act_c, const float4 *bq) {
            constexpr int ACT = decltype(act_c)::value;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const long long row = n0 + a_row + LN::RG * m;
                float *yrow = p.Y + row * p.out_f + colbase;
#pragma unroll
                for (int q = 0; q < TN / 4; ++q) {
                    float v[4] = {acc[m][2 * q].x, acc[m][2 * q].y, acc[m][2 * q + 1].x, acc[m][2 * q + 1].y};
                    if constexpr (DL >= 4) {
                        // v[e] = (k + e, l = r4) over lanes r4 = 0..3  ->  v[e] = (k + r4, l = e)
#pragma unroll
                        for (int t = 0; t < 2; ++t) {
                            const float snd = (r4 & 1) ? v[2 * t] : v[2 * t + 1];
                            const float rcv = __shfl_xor_sync(0xffffffffu, snd, 1);
                            if (r4 & 1) v[2 * t] = rcv; else v[2 * t + 1] = rcv;
                        }
#pragma unroll
                        for (int t = 0; t < 2; ++t) {
                            const float snd = (r4 & 2) ? v[t] : v[t + 2];
                            const float rcv = __shfl_xor_sync(0xffffffffu, snd, 2);
                            if (r4 & 2) v[t] = rcv; else v[t + 2] = rcv;
                        }
                    } else if constexpr (DL == 2) {
                        // lanes l = 0, 1 (lane bit 1): l = 0 takes (k, k+1) x (l0, l1), l = 1 takes (k+2, k+3)
                        const float s0 = c_l ? v[0] : v[2], s1 = c_l ? v[1] : v[3];
                        const float r0 = __shfl_xor_sync(0xffffffffu, s0, 2);
                        const float r1 = __shfl_xor_sync(0xffffffffu, s1, 2);
                        if (c_l) { v[0] = r0; v[1] = v[2]; v[2] = r1; }
                        else { v[3] = r1; v[2] = v[1]; v[1] = r0; }
                    }
                    if (bq) {
                        v[0] += bq[q].x; v[1] += bq[q].y; v[2] += bq[q].z; v[3] += bq[q].w;
                    }
                    ep_act4<ACT>(v);
                    const int k = kt + 4 * LN::KQ * q + k_off;  // first k of the vector
                    // the vector's four outputs are consecutive columns of Y (DL >= 4: (k, l_v + e);
                    // DL = 2 = d: (k + e/2, l0 + e%2); DL = 1: k + e)
                    if (row < p.N && k < p.b)
                        *reinterpret_cast<float4 *>(yrow + (long long)k * p.d) = make_float4(v[0], v[1], v[2], v[3]);
                }
            }
        };
        if (p.bias == nullptr && p.act == 0) {
            store_tile(std::integral_constant<int, 0>(), nullptr);
        } else {
            float4 bq[TN / 4];
#pragma unroll
            for (int q = 0; q < TN / 4; ++q) {
                const int k = kt + 4 * LN::KQ * q + k_off;
                const long long col = colbase + (long long)k * p.d;
                bq[q] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (p.bias && k < p.b) {
                    if (p.bias_vec4)
                        bq[q] = __ldg(reinterpret_cast<const float4 *>(p.bias + col));
                    else
                        bq[q] = make_float4(__ldg(p.bias + col), __ldg(p.bias + col + 1), __ldg(p.bias + col + 2),
                                            __ldg(p.bias + col + 3));
                }
            }
            const float4 *bp = p.bias ? bq : nullptr;
            switch (p.act) {
                case 1: store_tile(std::integral_constant<int, 1>(), bp); break;
                case 2: store_tile(std::integral_constant<int, 2>(), bp); break;
                case 3: store_tile(std::integral_constant<int, 3>(), bp); break;
                default: store_tile(std::integral_constant<int, 0>(), bp); break;
            }
        }
    }
}

template <int DL, int WM, int WK, int TN>
cudaError_t launch_cfg32(const Problem &pr, const float *vt) {
    using TL = Tile32<DL, WM, WK, TN>;
    Fma32Params p;
    p.X = static_cast<const float *>(pr.X);
    p.V = vt ? vt : static_cast<const float *>(pr.V);
    p.Y = static_cast<float *>(pr.Y);
    p.bias = static_cast<const float *>(pr.bias);
    p.bias_vec4 = (reinterpret_cast<uintptr_t>(pr.bias) % 16) == 0;
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
    const size_t smem = (size_t)((TL::SMEM_FLOATS * 4 + 15) / 16 * 16) + 2 * TL::NS * 8 + 16;
    if (smem > 232448) return cudaErrorInvalidConfiguration;
    p.status = device_status_ptr();
    if (!p.status) return cudaErrorUnknown;
    auto kern = vt ? fma32_kernel<DL, WM, WK, TN, true> : fma32_kernel<DL, WM, WK, TN, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = std::min<long long>(p.n_tiles, (long long)sm_count());
    kern<<<(int)grid, kThreads, smem, pr.stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

namespace {

// Tiles of this kernel (dl, wm, wk, tn): BM = 8*RG*wm rows, BKL = KQ*tn*wk k.
constexpr FmaConfig kFma32Configs[] = {
    {8, 2, 4, 16}, {8, 4, 2, 16}, {8, 2, 4, 12}, {8, 4, 2, 12},  // 64x64 128x32 64x48 128x24
    {4, 2, 4, 16}, {4, 1, 8, 16}, {4, 4, 2, 16}, {4, 2, 4, 12}, {4, 1, 8, 12},  // 128x64 64x128 256x32 128x48 64x96
    {2, 2, 4, 16}, {2, 4, 2, 16}, {2, 8, 1, 16}, {2, 2, 4, 12}, {2, 4, 2, 12},  // 128x128 256x64 512x32 128x96 256x48
    {1, 4, 2, 16}, {1, 8, 1, 16}, {1, 2, 4, 16}, {1, 4, 2, 12}, {1, 8, 1, 12},  // 256x128 512x64 128x256 256x96 512x48
};

int cfg_bm(const FmaConfig &c) { return 8 * (32 / (c.dl * (c.dl == 2 ? 2 : c.dl == 1 ? 4 : 1))) * c.wm; }
int cfg_bk(const FmaConfig &c) { return (c.dl == 2 ? 2 : c.dl == 1 ? 4 : 1) * c.tn * c.wk; }

// Tile choice: the fraction of SMs given a tile, discounted by the rows and k
// a partial tile wastes and by sqrt(TN/16) (the 12-k thread tiles issue more
// loads per FMA than the 16-k ones).  Every tile of the table keeps the FMA
// pipes fed once the SMs are full, so the staged-operand reuse BM*BKL/(BM+BKL)
// that an earlier rule rewarded picked tiles that left SMs idle or wasted rows;
// timed on every tile of the 258-pattern fp32 sweep at 25088 rows, this rule's
// pick is 0.3% slower than the fastest tile in the mean (23% at worst), the
// reuse rule's 2.5% (46% at worst).
FmaConfig fma32_choose(const Problem &p, int dl) {
    FmaConfig best = {0, 0, 0, 0};
    double best_score = -1.0;
    for (const FmaConfig &c : kFma32Configs) {
        if (c.dl != dl) continue;
        const int bm = cfg_bm(c), bkl = cfg_bk(c);
        const double kb = (double)((p.b + bkl - 1) / bkl);
        const double waste_k = kb * bkl / (double)p.b;
        const double rb = (double)((p.batch + bm - 1) / bm);
        const double waste_n = rb * bm / (double)p.batch;
        const double tiles = rb * kb * (double)(p.a * (p.d / dl));
        const double fill = std::min(1.0, tiles / (double)sm_count());
        const double score = std::sqrt(c.tn / 16.0) * fill / (waste_k * waste_n);
        if (score > best_score) { best_score = score; best = c; }
    }
    return best;
}

cudaError_t launch_cfg_any(const Problem &p, const FmaConfig &c, const float *vt) {
#define KS_FMA32_CASE(DL_, WM_, WK_, TN_) \
    if (c.dl == DL_ && c.wm == WM_ && c.wk == WK_ && c.tn == TN_) return launch_cfg32<DL_, WM_, WK_, TN_>(p, vt);
    KS_FMA32_CASE(8, 2, 4, 16)
    KS_FMA32_CASE(8, 4, 2, 16)
    KS_FMA32_CASE(8, 2, 4, 12)
    KS_FMA32_CASE(8, 4, 2, 12)
    KS_FMA32_CASE(4, 2, 4, 16)
    KS_FMA32_CASE(4, 1, 8, 16)
    KS_FMA32_CASE(4, 4, 2, 16)
    KS_FMA32_CASE(4, 2, 4, 12)
    KS_FMA32_CASE(4, 1, 8, 12)
    KS_FMA32_CASE(2, 2, 4, 16)
    KS_FMA32_CASE(2, 4, 2, 16)
    KS_FMA32_CASE(2, 8, 1, 16)
    KS_FMA32_CASE(2, 2, 4, 12)
    KS_FMA32_CASE(2, 4, 2, 12)
    KS_FMA32_CASE(1, 4, 2, 16)
    KS_FMA32_CASE(1, 8, 1, 16)
    KS_FMA32_CASE(1, 2, 4, 16)
    KS_FMA32_CASE(1, 4, 2, 12)
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
// If the workspace cannot be had, or the caller must not allocate
// (Problem::no_workspace), the values are read in place.
cudaError_t launch_fma32(const Problem &p, const FmaConfig &c_in) {
    // the l width comes from the caller's plan, the tile from this kernel's table
    const FmaConfig c = fma32_choose(p, c_in.dl);
    if (c.dl == 0) return cudaErrorInvalidConfiguration;
    const long long nvals = p.a * p.b * p.c * p.d;
    const double flops = 2.0 * (double)p.batch * (double)nvals;
    if (!p.no_workspace && c.dl == 8 && p.b % 4 == 0 && flops >= 1073741824.0 && nvals * 4 <= (64LL << 20)) {
        void *vt = nullptr;
        if (pool_alloc(&vt, (size_t)nvals * 4, p.stream) == cudaSuccess) {
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
