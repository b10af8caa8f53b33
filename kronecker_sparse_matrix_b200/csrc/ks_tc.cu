// tcgen05 tensor-core block-GEMM for KS products with bf16 inputs
// (fp32 accumulation in tensor memory, bf16 output rounded to nearest even).
//
// Y[n, i*b*d + k*d + l] = sum_{j<c} values[i, l, k, j] * X[n, i*c*d + j*d + l]
// (taxoreview.com page on Kronecker-sparse matrix multiplication, first
// abstract: a fused output-stationary kernel, no permutation passes).
//
// For one block i and offset l this is the dense GEMM
//     D_l[n, k] = sum_j A_l[n, j] * B_l[k, j],  A_l = X[:, i, :, l],  B_l = values[i, l]
// with M = 128 rows of the batch, N = the k of one pass, K = c.
//
// A tile is 128 rows x one block i x DLS consecutive l (DLS = 8 when d % 8 ==
// 0, else DLS = d).  Its outputs for all l and all k of a pass (DLS * bp <=
// 512 fp32 columns) accumulate in tensor memory while X streams through a
// ring of 16/32 KB chunks exactly once per pass; most patterns need a single
// pass, so X is read once and Y written once.  Each pass is its own tile, and
// the passes of one X tile are consecutive tiles, which run at the same time on
// neighbouring CTAs and share X through L2.
//
//   warp 0      TMA producer: raw X chunks (128 rows x 64..128 (j, l)
//               elements; l innermost, the only shape a tensor map can fetch
//               from the strided layout) into the ring, and the values of
//               the same j range into a 3..4-deep ring, as DLS K-major planes
//               whose rows (one k, the chunk's j) carry the swizzle of their
//               width (a TMA copy moves about one box row per clock, so the
//               rows are made as wide as the chunk allows);
//   warps 2..5  (DLS > 1) transpose each chunk in place, in registers, from
//               [row][j][l] to one MN-major no-swizzle operand plane per l,
//               row groups padded and skewed so every quarter-warp's 16-byte
//               accesses reach eight bank groups; for d = 1 the TMA box
//               already lands as the 128-byte-swizzled K-major tile the MMA
//               reads, and these warps idle;
//   warp 1      one thread issues tcgen05.mma (kind::f16, M=128, N=bp, K=16)
//               per plane and K step, commits to mbarriers;
//   warps 6..9  tcgen05.ld the accumulators (each warp its 32 TMEM lanes =
//               rows), round to bf16, interleave the l planes back into Y's
//               (k, l) order in a shared-memory staging box of 32 rows, and
//               hand it to a TMA tensor store when the box is contiguous in Y
//               (d == DLS), or copy it out in 16-byte stores otherwise.
//
// Every mbarrier wait is bounded (about one second of %globaltimer); a wait
// that runs out sets the device status word and raises the CTA's abort flag,
// every role drains its in-flight copies (bounded), and the CTA still frees
// its tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "ks_epilogue.cuh"
#include "ks_internal.h"
#include "ks_sm100.cuh"

namespace ks {
namespace {

using namespace sm100;

constexpr int kRows = 128;         // MMA M
constexpr int kStepJ = 16;         // j per MMA (bf16 K)
constexpr int kVStages = 4;        // values ring depth bound
constexpr int kMaxStages = 8;      // X ring depth bound
constexpr int kThreads = 320;      // 10 warps
constexpr int kLoadWarp0 = 2;      // warps 2..5
constexpr int kEpiWarp0 = 6;       // warps 6..9
constexpr int kEpiWarpBytes = 4096; // staging per epilogue warp: one box of 32 rows x 128 B
constexpr int kChunkElems = 64;     // output elements per row per epilogue chunk
constexpr int kSmemLimit = 232448; // per-block opt-in maximum on sm_100

// j per X chunk and chunk bytes, per DLS
__host__ __device__ constexpr int chunk_j(int dls) { return dls == 8 ? 16 : 64 / dls; }
__host__ __device__ constexpr int chunk_bytes(int dls) { return kRows * chunk_j(dls) * dls * 2; }
// Transposed operand planes (DLS > 1): MN-major core matrices of 8 j x 8 rows
// (128 bytes), the 16 row groups of a j octet 144 bytes apart (one 16-byte
// pad each), so that the transposer's 16-byte stores from one warp spread
// over all eight bank groups; j octets are 16 * 144 bytes apart.
constexpr int kGroupStride = 144;
constexpr int kOctetStride = 16 * kGroupStride;
// ring slot: the raw chunk, transposed in place into padded planes
__host__ __device__ constexpr int slot_bytes(int dls) {
    return dls == 1 ? chunk_bytes(1) : dls * (chunk_j(dls) / 8) * kOctetStride;
}
// The values of one chunk land as DLS planes of bp rows (k) x chunk_j(dls) j,
// K-major with the swizzle as wide as a row (2 * chunk_j bytes): tcgen05
// layout type and the TMA swizzle mode for that width.
__host__ __device__ constexpr uint32_t v_layout(int dls) {
    return chunk_j(dls) == 64 ? 2u : chunk_j(dls) == 32 ? 4u : 6u;
}

struct TcParams {
    const __nv_bfloat16 *bias;  // fused epilogue: out_f values or null
    int act;
    long long N;
    int a, b, c, d;
    int out_f;
    int bp, passes, n_g, kc, nbuf;
    long long n_tiles;
    __nv_bfloat16 *Y;
    unsigned *status;
    int stages;                      // X ring depth
    int vstages;                     // values ring depth
    int off_v, off_epi, off_bar;     // shared-memory carve-up (ring at offset 0)
    int v_stage_bytes;
    int box_elems, box_sw128;        // epilogue staging box: elements per row, swizzled
    int box_row_bytes;               // staging row stride when not swizzled (an odd number of 16-byte units)
    int ytma;                        // the swizzled staging box goes to Y as one TMA store (d == DLS)
    int x3d;                         // X chunks come from the (c*d, a, N) map (DLS < 8, or d == 8)
};

template <int DLS, bool EP>  // EP: fused bias / activation epilogue compiled in
__global__ void __launch_bounds__(kThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap vmap,
              const __grid_constant__ CUtensorMap ymap, const TcParams p) {
    constexpr int CTJ = chunk_j(DLS);
    constexpr int CB = chunk_bytes(DLS);
    constexpr int SB = slot_bytes(DLS);
    constexpr int UNITS = CTJ * DLS / 8;    // 16-byte units per row of a chunk (8 or 16)
    constexpr int TASKS = 16 * UNITS / 128; // transpose tasks per loader thread (1 or 2)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sR = smem;  // X ring: stage s at s * SB (1024-aligned)
    uint8_t *sV = smem + p.off_v;
    uint8_t *sE = smem + p.off_epi;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    uint64_t *x_full = bars;                   // [kMaxStages] TMA landed
    uint64_t *a_ready = x_full + kMaxStages;   // [kMaxStages] transposed in place
    uint64_t *x_empty = a_ready + kMaxStages;  // [kMaxStages] MMAs done with it
    uint64_t *v_full = x_empty + kMaxStages;   // [kVStages]
    uint64_t *v_empty = v_full + kVStages;     // [kVStages]
    uint64_t *acc_full = v_empty + kVStages;   // [2]
    uint64_t *acc_empty = acc_full + 2;        // [2]
    uint64_t *mma_done = acc_empty + 2;        // [1]
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_steps = p.c / kStepJ;
    const int n_chunks = (p.c + CTJ - 1) / CTJ;
    const int groups_per_i = p.d / DLS;
    const int S = p.stages;
    const int VS = p.vstages;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&a_ready[s], 128);
            mbar_init(&x_empty[s], 1);
        }
        for (int s = 0; s < kVStages; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
        for (int s = 0; s < 2; ++s) { mbar_init(&acc_full[s], 1); mbar_init(&acc_empty[s], 128); }
        mbar_init(mma_done, 1);
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
            uint32_t xq = 0, vq = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
                const int ps = (int)(tile % p.passes);
                const long long t2 = tile / p.passes;
                const int g = (int)(t2 % p.n_g);
                const long long rb = t2 / p.n_g;
                const int i = g / groups_per_i, l0 = (g % groups_per_i) * DLS;
                const int n0 = (int)(rb * kRows);
                {
                    for (int ch = 0; ch < n_chunks && ok; ++ch) {
                        const int xs = xq % S;
                        ok = mbar_wait(&x_empty[xs], ((xq / S) & 1) ^ 1, abort_flag, p.status);
                        if (!ok) break;
                        mbar_expect_tx(&x_full[xs], (uint32_t)CB);
                        if (DLS == 8 && !p.x3d)
                            tma_load_4d(sR + xs * SB, &xmap, &x_full[xs], l0, ch * CTJ, i, n0);
                        else
                            tma_load_3d(sR + xs * SB, &xmap, &x_full[xs], ch * CTJ * p.d, i, n0);
                        ++xq;  // counted as soon as it is in flight (the abort drain relies on it)
                        // the values of the same CTJ j: values[i, l0:l0+DLS, pass k's, chunk j's]
                        const int vs = vq % VS;
                        ok = mbar_wait(&v_empty[vs], ((vq / VS) & 1) ^ 1, abort_flag, p.status);
                        if (!ok) break;
                        mbar_expect_tx(&v_full[vs], (uint32_t)p.v_stage_bytes);
                        tma_load_3d(sV + vs * p.v_stage_bytes, &vmap, &v_full[vs], ch * CTJ, ps * p.bp, i * p.d + l0);
                        ++vq;
                    }
                }
            }
            // On abort, copies already issued may still be landing in shared
            // memory: wait (bounded) for them before leaving.
            if (*abort_flag) {
                for (uint32_t k = (xq >= (uint32_t)S ? xq - S : 0); k < xq; ++k)
                    mbar_wait_drain(&x_full[k % S], (k / S) & 1);
                for (uint32_t k = (vq >= (uint32_t)VS ? vq - VS : 0); k < vq; ++k)
                    mbar_wait_drain(&v_full[k % VS], (k / VS) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (one thread)
        if (lane == 0) {
            // kind::f16: D fp32 (bit 4), A and B bf16 (bits 7, 10), A MN-major
            // (bit 15) unless d == 1 (K-major), B K-major, N = bp, M = 128.
            const uint32_t a_major = (DLS == 1) ? 0u : 1u;
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (a_major << 15) |
                                   ((uint32_t)(p.bp >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
            uint32_t xq = 0, vq = 0, accq = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
                for (int once = 0; once < 1 && ok; ++once, ++accq) {
                    const int buf = (int)(accq % p.nbuf);
                    ok = mbar_wait(&acc_empty[buf], ((accq / p.nbuf) & 1) ^ 1, abort_flag, p.status);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t d_base = tmem_base + (uint32_t)(buf * DLS * p.bp);
                    for (int ch = 0; ch < n_chunks && ok; ++ch, ++xq) {
                        const int xs = xq % S;
                        // d == 1: the TMA tile is the operand; otherwise wait for the transpose
                        ok = mbar_wait(DLS == 1 ? &x_full[xs] : &a_ready[xs], (xq / S) & 1, abort_flag, p.status);
                        if (!ok) break;
                        const int vs = vq % VS;
                        ok = mbar_wait(&v_full[vs], (vq / VS) & 1, abort_flag, p.status);
                        ++vq;
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t stage = su32(sR) + xs * SB;
                        const uint32_t vstage = su32(sV) + vs * p.v_stage_bytes;
                        for (int s = ch * CTJ / kStepJ; s < n_steps && s < (ch + 1) * CTJ / kStepJ; ++s) {
                            const int sl = s - ch * CTJ / kStepJ;  // K step within the chunk
#pragma unroll
                            for (int l = 0; l < DLS; ++l) {
                                uint64_t ad;
                                if (DLS == 1)
                                    ad = smem_desc_sw128(stage + sl * 32, 1024);
                                else
                                    ad = smem_desc(stage + l * (CTJ / 8) * kOctetStride + sl * 2 * kOctetStride,
                                                   kOctetStride, kGroupStride);
                                // values stage: [l][bp k][CTJ j] swizzled rows, K step = 32 bytes
                                const uint32_t b_addr = vstage + l * (p.bp * CTJ * 2) + sl * 32;
                                const uint64_t bd = smem_desc_sw(b_addr, 8 * CTJ * 2, v_layout(DLS));
                                mma_bf16(d_base + l * p.bp, ad, bd, idesc, s > 0 ? 1u : 0u);
                            }
                        }
                        mma_commit(&v_empty[vs]);
                        mma_commit(&x_empty[xs]);
                    }
                    if (ok) mma_commit(&acc_full[buf]);
                }
            }
            // every MMA this thread issued has finished before TMEM is freed
            mma_commit(mma_done);
            mbar_wait_drain(mma_done, 0);
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------ in-place transpose (DLS > 1)
        if (DLS > 1) {
            const int t = threadIdx.x - kLoadWarp0 * 32;  // 0..127
            // task -> (16-byte unit q of a raw row, row group g8).  16-byte shared
            // accesses are served eight lanes at a time, so every eight
            // consecutive lanes must reach eight distinct bank groups, both when
            // reading the raw chunk (group = q) and when writing the padded planes
            // (group = g8 + the unit's j mod 8); for two and four l the row group
            // is skewed by the unit for that.
            auto task_unit = [&](int task, int &q, int &g8) {
                if (DLS == 8) {
                    q = task % UNITS;
                    g8 = task / UNITS;
                } else {
                    q = task & 7;
                    g8 = ((task >> 3) + (q >> (DLS == 2 ? 1 : 2))) & 15;
                }
            };
            uint32_t xq = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
                {
                    for (int ch = 0; ch < n_chunks; ++ch, ++xq) {
                        const int xs = xq % S;
                        const bool w = mbar_wait(&x_full[xs], (xq / S) & 1, abort_flag, p.status);
                        ok = bar_and(1, 128, w);  // uniform over the four loader warps
                        if (!ok) break;
                        uint8_t *st = sR + xs * SB;
                        uint4 out[TASKS][8];
#pragma unroll
                        for (int k = 0; k < TASKS; ++k) {
                            int q, g8;
                            task_unit(t + 128 * k, q, g8);
                            uint4 in[8];
#pragma unroll
                            for (int r = 0; r < 8; ++r)
                                in[r] = *reinterpret_cast<const uint4 *>(st + ((g8 * 8 + r) * UNITS + q) * 16);
                            transpose8x8_b16(in, out[k]);
                        }
                        bar_sync(1, 128);  // every read of the raw chunk is done
#pragma unroll
                        for (int k = 0; k < TASKS; ++k) {
                            int q, g8;
                            task_unit(t + 128 * k, q, g8);
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int f = 8 * q + e;
                                const int j = f / DLS, l = f % DLS;  // j within the chunk
                                *reinterpret_cast<uint4 *>(st + (l * (CTJ / 8) + (j >> 3)) * kOctetStride +
                                                           g8 * kGroupStride + (j & 7) * 16) = out[k][e];
                            }
                        }
                        fence_proxy_async();
                        mbar_arrive(&a_ready[xs]);
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue: TMEM -> bf16 -> Y
        // Per output chunk (kc k's, DLS*kc <= 64 elements per row): tcgen05.ld
        // the warp's 32 rows, round to bf16 in (k, l) order, write the rows into
        // a staging box (128-byte rows with the 16-byte units XOR-swizzled by
        // row when the row holds 64 elements: conflict-free 16-byte stores and
        // loads), then copy the box to Y, four full 128-byte row segments per
        // warp instruction.
        const int ew = warp - kEpiWarp0;          // 0..3
        const int quad = warp & 3;                // TMEM lanes 32*quad .. 32*quad+31
        uint8_t *stage = sE + ew * kEpiWarpBytes; // 1024-aligned
        const int kc = p.kc;                      // k per chunk
        const int n_oc = p.bp / kc;
        const int units = DLS * kc / 8;           // 16-byte output units per row per chunk
        const bool sw = p.box_sw128 != 0;
        // staging row stride (not sw): dense rows for the tensor store, else padded rows
        const int rsb = p.ytma ? p.box_elems * 2 : p.box_row_bytes;
        uint32_t accq = 0;
        bool ok = true;
        for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
            const int ps = (int)(tile % p.passes);
            const long long t2 = tile / p.passes;
            const int g = (int)(t2 % p.n_g);
            const long long rb = t2 / p.n_g;
            const int i = g / groups_per_i, l0 = (g % groups_per_i) * DLS;
            const int row0 = (int)(rb * kRows) + 32 * quad;
            for (int once = 0; once < 1 && ok; ++once, ++accq) {
                const int buf = (int)(accq % p.nbuf);
                ok = mbar_wait(&acc_full[buf], (accq / p.nbuf) & 1, abort_flag, p.status);
                ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
                if (!ok) break;
                tc_fence_after();
                for (int oc = 0; oc < n_oc; ++oc) {
                    float acc[DLS][kChunkElems / DLS];
#pragma unroll
                    for (int l = 0; l < DLS; ++l) {
#pragma unroll
                        for (int pc = 0; pc < kChunkElems / DLS / 8; ++pc) {
                            if (pc * 8 < kc) {
                                float v[8];
                                const uint32_t col = (uint32_t)(buf * DLS * p.bp + l * p.bp + oc * kc + pc * 8);
                                tmem_ld8(tmem_base + ((uint32_t)(32 * quad) << 16) + col, v);
#pragma unroll
                                for (int qq = 0; qq < 8; ++qq) acc[l][pc * 8 + qq] = v[qq];
                            }
                        }
                    }
                    tmem_ld_wait();
                    if (oc == n_oc - 1) {  // accumulator buffer no longer needed: hand it back
                        tc_fence_before();
                        mbar_arrive(&acc_empty[buf]);
                    }
                    const int kq = ps * p.bp + oc * kc;  // first k of the chunk
                    const long long ybase = (long long)i * p.b * p.d + l0;
                    if (EP && p.bias) {  // fused epilogue on (k = kq + e, l)
#pragma unroll
                        for (int l = 0; l < DLS; ++l)
#pragma unroll
                            for (int e = 0; e < kChunkElems / DLS; ++e)
                                if (e < kc) acc[l][e] += ep_bias(p.bias, ybase + (long long)(kq + e) * p.d + l);
                    }
                    if (EP && p.act) {
#pragma unroll
                        for (int l = 0; l < DLS; ++l) ep_act_array(acc[l], p.act);
                    }
                    if (p.ytma) {  // the previous box store has finished reading the staging
                        if (lane == 0) bulk_wait_read_all();
                        __syncwarp();
                    }
                    // unit u = elements 8u..8u+7 of (k*DLS + l); box u*8/bi, 16-byte chunk within its row
#pragma unroll
                    for (int u = 0; u < kChunkElems / 8; ++u) {
                        if (u < units) {
                            uint32_t w[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const int f0 = 8 * u + 2 * h, f1 = f0 + 1;
                                w[h] = pack_bf16x2(acc[f0 % DLS][f0 / DLS], acc[f1 % DLS][f1 / DLS]);
                            }
                            const uint32_t off = sw ? lane * 128 + ((u ^ (lane & 7)) << 4) : lane * rsb + u * 16;
                            *reinterpret_cast<uint4 *>(stage + off) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                    if (p.ytma) {
                        // d == DLS: the box is 32 rows x DLS*kc contiguous elements of Y at column
                        // ybase + kq*d (staged in the TMA's 128-byte swizzle when rows are 128 bytes,
                        // densely otherwise); one thread hands it to the tensor store (rows past N
                        // are clipped by the tensor map)
                        fence_proxy_async();
                        __syncwarp();
                        if (lane == 0 && (long long)row0 < p.N) {
                            tma_store_2d(&ymap, su32(stage), (int)(ybase + (long long)kq * p.d), row0);
                            bulk_commit();
                        }
                        continue;
                    }
                    __syncwarp();
                    // copy the box out: lane = (row r = lane / 8 + 4 t, unit u = lane % 8), so each
                    // warp instruction moves whole 16-byte units of four rows (four full 128-byte row
                    // segments when sw); lanes past the row's units idle
                    {
                        const int u = lane & 7;
                        if (u < units) {
                            const int f = 8 * u;
                            const long long col = ybase + (long long)(kq + f / DLS) * p.d + f % DLS;
                            int r = lane >> 3;
                            __nv_bfloat16 *yp = p.Y + (long long)(row0 + r) * p.out_f + col;
                            const long long ystep = 4LL * p.out_f;
                            const int rows_here = (int)min(p.N - (long long)row0, 32LL);
#pragma unroll
                            for (int t = 0; t < 8; ++t, r += 4, yp += ystep) {
                                if (r < rows_here) {
                                    const uint32_t soff = sw ? r * 128 + ((u ^ (r & 7)) << 4) : r * rsb + u * 16;
                                    *reinterpret_cast<uint4 *>(yp) = *reinterpret_cast<const uint4 *>(stage + soff);
                                }
                            }
                        }
                    }
                    __syncwarp();
                }
            }
        }
    }

    // the box stores issued by this warp's lane 0 are complete before the CTA
    // (and its shared memory) goes away
    if (warp >= kEpiWarp0 && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

int tc_dls(const Problem &p) {
    if (p.d % 8 == 0) return 8;
    if (p.d == 1 || p.d == 2 || p.d == 4) return (int)p.d;
    return 0;
}

// k per epilogue chunk: a multiple of 8 dividing bp with dls * kc <= 64,
// preferring rows of exactly 64 elements (one 128-byte swizzled store box).
int tc_kc(int dls, int bp) {
    for (int kc = std::min(bp, kChunkElems / dls); kc >= 8; kc -= 8)
        if (bp % kc == 0 && dls * kc == kChunkElems) return kc;
    for (int kc = std::min(bp, kChunkElems / dls); kc >= 8; kc -= 8)
        if (bp % kc == 0) return kc;
    return 0;
}

// k per pass: the largest multiple of 16 dividing b with dls * bp <= 512 and
// bp <= 256 (a single accumulator buffer when dls * bp > 256; smaller passes
// that fit twice were measured slower: every extra pass repeats the transpose
// of each X chunk).
int tc_bp(int dls, int64_t b) {
    for (int bp = std::min(256, 512 / dls); bp >= 16; bp -= 16)
        if (b % bp == 0) return bp;
    return 0;
}

struct TcLayout {
    int stages, vstages, v_stage_bytes, off_v, off_epi, off_bar, total;
};

constexpr int kBarBytes = (3 * kMaxStages + 2 * kVStages + 2 + 2 + 1) * 8 + 16;

// Shared memory: the X ring (as deep as fits, 3..8 chunks), the values ring
// (one stage per X chunk: DLS planes x bp k x CTJ j, 3..4 deep), the epilogue
// staging, barriers.
bool tc_layout(int dls, int bp, TcLayout *out) {
    TcLayout L;
    auto up = [](int x, int a) { return (x + a - 1) / a * a; };
    const int cb = slot_bytes(dls);
    L.v_stage_bytes = 2 * bp * chunk_j(dls) * dls;
    const int epi = 4 * kEpiWarpBytes;
    const int budget = kSmemLimit - 2048 - epi - kBarBytes;  // alignment slack
    L.vstages = (kVStages * L.v_stage_bytes + 3 * cb <= budget) ? kVStages : 3;
    const int left = budget - up(L.vstages * L.v_stage_bytes, 128);
    L.stages = std::min(kMaxStages, left / cb);
    if (L.stages < 2) return false;
    L.off_v = L.stages * cb;
    L.off_epi = up(L.off_v + L.vstages * L.v_stage_bytes, 1024);
    L.off_bar = up(L.off_epi + epi, 128);
    L.total = L.off_bar + kBarBytes + 1024;
    if (L.total > kSmemLimit) return false;
    *out = L;
    return true;
}

}  // namespace

TcConfig tc_choose(const Problem &p) {
    const int dls = tc_dls(p);
    TcConfig c{dls, 0, kStepJ};
    if (dls) c.bk = tc_bp(dls, p.b);
    return c;
}

bool tc_supported(const Problem &p, const char **why) {
    if (p.dtype != KS_BF16) { *why = "tensor-core kernel serves bf16"; return false; }
    const int dls = tc_dls(p);
    if (!dls) { *why = "d must be 1, 2, 4 or a multiple of 8"; return false; }
    if (p.c % kStepJ) { *why = "c must be a multiple of 16"; return false; }
    const uintptr_t al = reinterpret_cast<uintptr_t>(p.X) | reinterpret_cast<uintptr_t>(p.V) |
                         reinterpret_cast<uintptr_t>(p.Y);
    if (al % 16) { *why = "X, values and Y must be 16-byte aligned"; return false; }
    const int bp = tc_bp(dls, p.b);
    TcLayout L;
    if (bp == 0 || tc_kc(dls, bp) == 0) { *why = "b has no pass width (a multiple of 16 dividing it)"; return false; }
    if (!tc_layout(dls, bp, &L)) { *why = "shared memory budget"; return false; }
    if (p.batch > (1LL << 31) - 256 || p.a * p.d > (1LL << 31)) { *why = "sizes exceed tensor-map coordinates"; return false; }
    return true;
}

template <int DLS>
static cudaError_t launch_dls(const Problem &pr, const TcConfig &cfg) {
    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    const int bp = cfg.bk;
    TcLayout L;
    if (bp == 0 || !tc_layout(DLS, bp, &L)) return cudaErrorInvalidConfiguration;
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUtensorMap xmap, vmap;
    CUresult r;
    const bool x3d = DLS < 8 || pr.d == 8;
    if (!x3d) {
        // X as (d, c, a, N): a box (8 l, 16 j, 1, 128 rows) = [row][j][l]
        cuuint64_t dims[4] = {(cuuint64_t)pr.d, (cuuint64_t)pr.c, (cuuint64_t)pr.a, (cuuint64_t)pr.batch};
        cuuint64_t strides[3] = {(cuuint64_t)pr.d * 2, (cuuint64_t)pr.c * pr.d * 2, (cuuint64_t)pr.in_features() * 2};
        cuuint32_t box[4] = {8, (cuuint32_t)chunk_j(8), 1, (cuuint32_t)kRows};
        r = encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(pr.X), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        // X as (c*d, a, N): a box (CTJ*DLS elements, 1, 128 rows) = [row][(j, l)]
        // (d == DLS, or d == 8: whole 256-byte rows); for d == 1 with the
        // 128-byte swizzle, the K-major operand tile itself
        cuuint64_t dims[3] = {(cuuint64_t)(pr.c * pr.d), (cuuint64_t)pr.a, (cuuint64_t)pr.batch};
        cuuint64_t strides[2] = {(cuuint64_t)pr.c * pr.d * 2, (cuuint64_t)pr.in_features() * 2};
        cuuint32_t box[3] = {(cuuint32_t)(chunk_j(DLS) * DLS), 1, (cuuint32_t)kRows};
        r = encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(pr.X), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, DLS == 1 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    {
        // values[i][l][k][j] viewed as (j, k, i*d+l): a box (CTJ j, bp k, DLS l)
        // lands as DLS planes [k][CTJ j], rows of 2*CTJ bytes swizzled at that
        // width: the K-major operand for CTJ/16 K steps.  (A TMA fetches about
        // one box row per clock, so rows of 16 bytes would cap the copy far
        // below the bandwidth this kernel needs.)
        cuuint64_t dims[3] = {(cuuint64_t)pr.c, (cuuint64_t)pr.b, (cuuint64_t)(pr.a * pr.d)};
        cuuint64_t strides[2] = {(cuuint64_t)pr.c * 2, (cuuint64_t)pr.b * pr.c * 2};
        cuuint32_t box[3] = {(cuuint32_t)chunk_j(DLS), (cuuint32_t)bp, (cuuint32_t)DLS};
        const CUtensorMapSwizzle vsw = chunk_j(DLS) == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                       : chunk_j(DLS) == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                            : CU_TENSOR_MAP_SWIZZLE_32B;
        r = encode(&vmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(pr.V), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, vsw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    // epilogue chunk: kc k's; rows of 64 elements use the swizzled staging box
    const int kc0 = tc_kc(DLS, bp);
    const bool ytma = pr.d == DLS && (reinterpret_cast<uintptr_t>(pr.Y) % 16) == 0;
    CUtensorMap ymap;
    memset(&ymap, 0, sizeof(ymap));
    if (ytma) {
        // Y as (out_f, N): a box (DLS*kc elements, 32 rows); 64-element rows with the
        // 128-byte swizzle of the staging, shorter rows packed densely
        const bool sw = DLS * kc0 == kChunkElems;
        cuuint64_t dims[2] = {(cuuint64_t)pr.out_features(), (cuuint64_t)pr.batch};
        cuuint64_t strides[1] = {(cuuint64_t)pr.out_features() * 2};
        cuuint32_t box[2] = {(cuuint32_t)(DLS * kc0), 32};
        r = encode(&ymap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pr.Y, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    const int kc = tc_kc(DLS, bp);
    if (kc == 0) return cudaErrorInvalidConfiguration;
    const bool sw128 = (DLS * kc) == kChunkElems;
    const int bi = DLS * kc;

    TcParams p;
    p.box_elems = bi;
    p.box_sw128 = sw128 ? 1 : 0;
    p.box_row_bytes = bi * 2 + ((bi / 8) % 2 == 0 ? 16 : 0);
    p.ytma = ytma ? 1 : 0;
    p.x3d = x3d ? 1 : 0;
    p.N = pr.batch;
    p.bias = static_cast<const __nv_bfloat16 *>(pr.bias);
    p.act = pr.act;
    p.a = (int)pr.a; p.b = (int)pr.b; p.c = (int)pr.c; p.d = (int)pr.d;
    p.out_f = (int)pr.out_features();
    p.bp = bp;
    p.passes = (int)(pr.b / bp);
    p.n_g = (int)(pr.a * (pr.d / DLS));
    p.kc = kc;
    p.nbuf = (2 * DLS * bp <= 512) ? 2 : 1;
    if (p.kc == 0) return cudaErrorInvalidConfiguration;
    // tiles = (row block, l group, pass of k), the pass varying fastest: CTAs
    // that run side by side take the passes of the same X tile, so its second
    // read is served by L2
    p.n_tiles = ((pr.batch + kRows - 1) / kRows) * p.n_g * p.passes;
    p.Y = static_cast<__nv_bfloat16 *>(pr.Y);
    p.status = device_status_ptr();
    if (!p.status) return cudaErrorUnknown;
    p.stages = L.stages;
    p.vstages = L.vstages;
    p.off_v = L.off_v;
    p.off_epi = L.off_epi;
    p.off_bar = L.off_bar;
    p.v_stage_bytes = L.v_stage_bytes;
    auto kern = (pr.bias || pr.act) ? tc_kernel<DLS, true> : tc_kernel<DLS, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (e != cudaSuccess) return e;
    const long long grid = std::min<long long>(p.n_tiles, (long long)sm_count());
    kern<<<(int)grid, kThreads, L.total, pr.stream>>>(xmap, vmap, ymap, p);
    return cudaGetLastError();
}

cudaError_t launch_tc(const Problem &p, const TcConfig &cfg) {
    switch (cfg.dl) {
        case 8: return launch_dls<8>(p, cfg);
        case 4: return launch_dls<4>(p, cfg);
        case 2: return launch_dls<2>(p, cfg);
        case 1: return launch_dls<1>(p, cfg);
        default: return cudaErrorInvalidConfiguration;
    }
}

}  // namespace ks
