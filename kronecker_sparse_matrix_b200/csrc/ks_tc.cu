// tcgen05 tensor-core block-GEMM for KS products with bf16 inputs
// (fp32 accumulation in tensor memory, bf16 output rounded to nearest even).
//
// Y[n, i*b*d + k*d + l] = sum_{j<c} values[i, l, k, j] * X[n, i*c*d + j*d + l]
// (taxoreview.com page on Kronecker-sparse matrix multiplication, first
// abstract: a fused output-stationary kernel, no permutation passes).
//
// For one block i and offset l this is the dense GEMM
//     D_l[n, k] = sum_j A_l[n, j] * B_l[k, j],  A_l = X[:, i, :, l],  B_l = values[i, l]
// with M = 128 rows of the batch, N = BK values of k and K = c.
//
// One CTA owns 128 rows x one block i x DLS consecutive l (DLS = 8 when
// d % 8 == 0, else DLS = d), and produces every k for them, so X is read from
// HBM once and Y written once:
//
//   warp 0      TMA: raw X chunks [128 rows][8 j][DLS l] (16-byte runs of l
//               innermost, the only shape a tensor map can fetch) into a
//               2-deep ring;
//   warps 2..5  transpose each chunk in registers (8 rows x 8 elements of
//               16 bits) into one MN-major no-swizzle operand plane per l,
//               resident for the whole tile, and stage values[i, l, k-block,
//               16 j] as K-major no-swizzle B tiles in a 4-deep ring;
//   warp 1      one elected thread issues tcgen05.mma (kind::f16, M=128,
//               N=BK, K=16) per plane and K step into a double-buffered TMEM
//               accumulator (DLS * BK fp32 columns per buffer), and commits
//               to mbarriers;
//   warps 6..9  tcgen05.ld the accumulators (each warp its 32 TMEM lanes =
//               rows), round to bf16, interleave the l planes back into
//               Y's (k, l) order through shared memory and store 16-byte
//               units, coalesced along each row.
//
// Every mbarrier wait is bounded (about one second of %globaltimer); a wait
// that runs out sets the device status word, raises the CTA's abort flag so
// that every role drains, and the CTA still frees its TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "ks_internal.h"

namespace ks {
namespace {

constexpr int kRows = 128;          // MMA M
constexpr int kChunkJ = 8;          // j per raw X chunk
constexpr int kStepJ = 16;          // j per MMA (bf16 K)
constexpr int kVStages = 4;
constexpr int kXStages = 2;
constexpr int kThreads = 320;       // 10 warps
constexpr int kLoadWarp0 = 2;       // warps 2..5
constexpr int kEpiWarp0 = 6;        // warps 6..9
constexpr int kEpiRowBytes = 272;   // 256 B of output + 16 B pad per staged row
constexpr int kMaxSteps = 32;       // c <= 512
constexpr uint64_t kTimeoutNs = 1000000000ull;

struct TcParams {
    const __nv_bfloat16 *V;
    __nv_bfloat16 *Y;
    long long N;
    int a, b, c, d;
    int in_f, out_f;
    int bk, nkb, n_g, kc;
    long long n_tiles;
    unsigned *status;
    // shared-memory carve-up (byte offsets from the aligned base)
    int off_a, off_v, off_x, off_epi, off_bar;
    int a_plane_bytes, v_stage_bytes, x_stage_bytes;
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t su32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(su32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Waits for the phase of `parity` to complete.  Returns false if the CTA is
// aborting or the wait ran out (which starts the abort).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          unsigned *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kTimeoutNs) {
            *abort_flag = 1;
            atomicOr(status, kDevTimeout);
            return false;
        }
    }
}
// Bounded wait used on the way out (ignores the abort flag).
__device__ __forceinline__ void mbar_wait_drain(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > kTimeoutNs) break;
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1, int c2,
                                            int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::
            "r"(su32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(su32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
            "r"(su32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(su32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t *holder, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(holder)), "r"(cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols));
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(bar))
                 : "memory");
}
// 16 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int q = 0; q < 16; ++q) v[q] = __uint_as_float(r[q]);
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, no swizzle (tcgen05 format: start, LBO,
// SBO in 16-byte units; bits 46-47 = 1).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// 8x8 transpose of 16-bit elements: in[s] holds elements e=0..7 of row s;
// out[e] holds rows s=0..7 of element e.
__device__ __forceinline__ void transpose8x8_b16(const uint4 (&in)[8], uint4 (&out)[8]) {
    uint32_t t[4][8];  // t[p][e]: (row 2p at e, row 2p+1 at e)
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint32_t a[4] = {in[2 * p].x, in[2 * p].y, in[2 * p].z, in[2 * p].w};
        const uint32_t b[4] = {in[2 * p + 1].x, in[2 * p + 1].y, in[2 * p + 1].z, in[2 * p + 1].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            t[p][2 * w] = __byte_perm(a[w], b[w], 0x5410);
            t[p][2 * w + 1] = __byte_perm(a[w], b[w], 0x7632);
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = make_uint4(t[0][e], t[1][e], t[2][e], t[3][e]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// ---------------------------------------------------------------- the kernel
template <int DLS>
__global__ void __launch_bounds__(kThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap xmap, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t *sA = smem + p.off_a;
    uint8_t *sV = smem + p.off_v;
    uint8_t *sX = smem + p.off_x;
    uint8_t *sE = smem + p.off_epi;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    uint64_t *x_full = bars;                       // [2]
    uint64_t *x_empty = bars + 2;                  // [2]
    uint64_t *v_full = bars + 4;                   // [4]
    uint64_t *v_empty = bars + 8;                  // [4]
    uint64_t *acc_full = bars + 12;                // [2]
    uint64_t *acc_empty = bars + 14;               // [2]
    uint64_t *a_free = bars + 16;                  // [1]
    uint64_t *mma_done = bars + 17;                // [1]
    uint64_t *a_ready = bars + 18;                 // [kMaxSteps]
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 18 + kMaxSteps);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_steps = p.c / kStepJ;
    const int n_chunks = p.c / kChunkJ;
    const int groups_per_i = p.d / DLS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kXStages; ++s) { mbar_init(&x_full[s], 1); mbar_init(&x_empty[s], 128); }
        for (int s = 0; s < kVStages; ++s) { mbar_init(&v_full[s], 128); mbar_init(&v_empty[s], 1); }
        for (int s = 0; s < 2; ++s) { mbar_init(&acc_full[s], 1); mbar_init(&acc_empty[s], 128); }
        mbar_init(a_free, 1);
        mbar_init(mma_done, 1);
        for (int s = 0; s < kMaxSteps; ++s) mbar_init(&a_ready[s], 128);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(tmem_holder, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t q = 0;  // global chunk counter
            for (long long tile = blockIdx.x; tile < p.n_tiles && !*abort_flag; tile += gridDim.x) {
                const int g = (int)(tile % p.n_g);
                const long long rb = tile / p.n_g;
                const int i = g / groups_per_i, l0 = (g % groups_per_i) * DLS;
                const int n0 = (int)(rb * kRows);
                for (int ch = 0; ch < n_chunks; ++ch, ++q) {
                    const int s = q % kXStages;
                    if (!mbar_wait(&x_empty[s], ((q / kXStages) & 1) ^ 1, abort_flag, p.status)) break;
                    mbar_expect_tx(&x_full[s], (uint32_t)p.x_stage_bytes);
                    if (DLS == 8 && p.d % 8 == 0)
                        tma_load_4d(sX + s * p.x_stage_bytes, &xmap, &x_full[s], l0, ch * kChunkJ, i, n0);
                    else
                        tma_load_3d(sX + s * p.x_stage_bytes, &xmap, &x_full[s], ch * kChunkJ * p.d, i, n0);
                }
            }
            // On abort, loads already issued may still be landing in shared
            // memory: wait (bounded) for the last ones before leaving.
            if (*abort_flag)
                for (uint32_t k = (q >= kXStages ? q - kXStages : 0); k < q; ++k)
                    mbar_wait_drain(&x_full[k % kXStages], (k / kXStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (one thread)
        if (lane == 0) {
        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((uint32_t)(p.bk >> 3) << 17) |
                               ((uint32_t)(kRows >> 4) << 24);
        uint32_t vq = 0, accq = 0, it = 0;
        for (long long tile = blockIdx.x; tile < p.n_tiles && !*abort_flag; tile += gridDim.x, ++it) {
            bool ok = true;
            for (int kb = 0; kb < p.nkb && ok; ++kb, ++accq) {
                const int buf = accq & 1;
                ok = mbar_wait(&acc_empty[buf], ((accq >> 1) & 1) ^ 1, abort_flag, p.status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d_base = tmem_base + (uint32_t)(buf * DLS * p.bk);
                for (int s = 0; s < n_steps; ++s, ++vq) {
                    const int vs = vq % kVStages;
                    ok = mbar_wait(&v_full[vs], (vq / kVStages) & 1, abort_flag, p.status);
                    if (ok && kb == 0) ok = mbar_wait(&a_ready[s], it & 1, abort_flag, p.status);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int l = 0; l < DLS; ++l) {
                        const uint32_t a_addr = su32(sA) + l * p.a_plane_bytes + s * 2 * 2048;
                        const uint32_t b_addr = su32(sV) + vs * p.v_stage_bytes + l * (p.bk * 32);
                        const uint64_t ad = smem_desc(a_addr, 2048, 128);
                        const uint64_t bd = smem_desc(b_addr, p.bk * 16, 128);
                        mma_bf16(d_base + l * p.bk, ad, bd, idesc, s > 0 ? 1u : 0u);
                    }
                    mma_commit(&v_empty[vs]);
                    if (s == n_steps - 1) {
                        mma_commit(&acc_full[buf]);
                        if (kb == p.nkb - 1) mma_commit(a_free);
                    }
                }
            }
        }
        // every MMA this thread issued has finished before TMEM is freed
        mma_commit(mma_done);
        mbar_wait_drain(mma_done, 0);
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------ loaders: X repack + values staging
        const int t = threadIdx.x - kLoadWarp0 * 32;  // 0..127
        uint32_t xq = 0, vq = 0, it = 0;
        for (long long tile = blockIdx.x; tile < p.n_tiles && !*abort_flag; tile += gridDim.x, ++it) {
            const int g = (int)(tile % p.n_g);
            const int i = g / groups_per_i, l0 = (g % groups_per_i) * DLS;
            bool ok = mbar_wait(a_free, (it & 1) ^ 1, abort_flag, p.status);
            for (int kb = 0; kb < p.nkb && ok; ++kb) {
                const int k0 = kb * p.bk;
                for (int s = 0; s < n_steps && ok; ++s, ++vq) {
                    // values[i, l0+l, k0:k0+bk, 16s:16s+16] -> K-major tile of plane l
                    const int vs = vq % kVStages;
                    ok = mbar_wait(&v_empty[vs], ((vq / kVStages) & 1) ^ 1, abort_flag, p.status);
                    if (!ok) break;
                    uint8_t *vdst = sV + vs * p.v_stage_bytes;
                    const int units = DLS * p.bk * 2;
                    for (int u = t; u < units; u += 128) {
                        const int k = u % p.bk;
                        const int rest = u / p.bk;
                        const int jc = rest & 1, l = rest >> 1;
                        const __nv_bfloat16 *src =
                            p.V + ((long long)(i * p.d + l0 + l) * p.b + (k0 + k)) * p.c + s * kStepJ + jc * 8;
                        const uint4 val = __ldg(reinterpret_cast<const uint4 *>(src));
                        *reinterpret_cast<uint4 *>(vdst + l * (p.bk * 32) + jc * (p.bk * 16) + k * 16) = val;
                    }
                    fence_proxy_async();
                    mbar_arrive(&v_full[vs]);
                    if (kb == 0) {
                        // the two raw X chunks of this K step -> operand planes
                        for (int h = 0; h < 2 && ok; ++h, ++xq) {
                            const int xs = xq % kXStages;
                            ok = mbar_wait(&x_full[xs], (xq / kXStages) & 1, abort_flag, p.status);
                            if (!ok) break;
                            const uint8_t *raw = sX + xs * p.x_stage_bytes;
                            const int jbase = (2 * s + h) * kChunkJ;
                            // task (row group g8, 16-byte unit q): 16 * DLS tasks
                            for (int task = t; task < 16 * DLS; task += 128) {
                                const int q = task % DLS, g8 = task / DLS;
                                uint4 in[8], out[8];
#pragma unroll
                                for (int r = 0; r < 8; ++r)
                                    in[r] = *reinterpret_cast<const uint4 *>(raw + ((g8 * 8 + r) * DLS + q) * 16);
                                transpose8x8_b16(in, out);
#pragma unroll
                                for (int e = 0; e < 8; ++e) {
                                    const int f = 8 * q + e;  // element within the row's chunk: (j, l)
                                    const int jl = f / DLS, ll = f % DLS;
                                    const int j = jbase + jl;
                                    *reinterpret_cast<uint4 *>(sA + ll * p.a_plane_bytes + (j >> 3) * 2048 + g8 * 128 +
                                                               (j & 7) * 16) = out[e];
                                }
                            }
                            mbar_arrive(&x_empty[xs]);
                        }
                        fence_proxy_async();
                        mbar_arrive(&a_ready[s]);
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue: TMEM -> bf16 -> Y
        const int ew = warp - kEpiWarp0;          // 0..3
        const int quad = warp & 3;                // TMEM lanes 32*quad .. 32*quad+31
        uint8_t *stage = sE + ew * 32 * kEpiRowBytes;
        const int kc = p.kc;                      // k per chunk (divides bk, DLS*kc <= 128)
        const int n_ch = p.bk / kc;
        const int units = DLS * kc / 8;           // 16-byte output units per row per chunk
        uint32_t accq = 0;
        for (long long tile = blockIdx.x; tile < p.n_tiles && !*abort_flag; tile += gridDim.x) {
            const int g = (int)(tile % p.n_g);
            const long long rb = tile / p.n_g;
            const int i = g / groups_per_i, l0 = (g % groups_per_i) * DLS;
            const long long row0 = rb * kRows + 32 * quad;
            bool ok = true;
            for (int kb = 0; kb < p.nkb && ok; ++kb, ++accq) {
                const int buf = accq & 1;
                ok = mbar_wait(&acc_full[buf], (accq >> 1) & 1, abort_flag, p.status);
                ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
                if (!ok) break;
                tc_fence_after();
                for (int ch = 0; ch < n_ch; ++ch) {
                    float acc[DLS][128 / DLS];
#pragma unroll
                    for (int l = 0; l < DLS; ++l) {
#pragma unroll
                        for (int pc = 0; pc < 128 / DLS / 16; ++pc) {
                            if (pc * 16 < kc) {
                                float v[16];
                                const uint32_t col = (uint32_t)(buf * DLS * p.bk + l * p.bk + ch * kc + pc * 16);
                                tmem_ld16(tmem_base + ((uint32_t)(32 * quad) << 16) + col, v);
#pragma unroll
                                for (int q = 0; q < 16; ++q) acc[l][pc * 16 + q] = v[q];
                            }
                        }
                    }
                    tmem_ld_wait();
                    // interleave (k, l) into 16-byte units: unit u = elements 8u..8u+7 of (k*DLS + l)
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        if (u < units) {
                            uint32_t w[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const int f0 = 8 * u + 2 * h, f1 = f0 + 1;
                                w[h] = pack_bf16x2(acc[f0 % DLS][f0 / DLS], acc[f1 % DLS][f1 / DLS]);
                            }
                            *reinterpret_cast<uint4 *>(stage + lane * kEpiRowBytes + u * 16) =
                                make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                    __syncwarp();
                    // copy out: row r of this warp, unit u -> Y[row, i, k, l]
                    for (int idx = lane; idx < 32 * units; idx += 32) {
                        const int r = idx / units, u = idx % units;
                        const long long row = row0 + r;
                        if (row < p.N) {
                            const int f = 8 * u;
                            const int k = kb * p.bk + ch * kc + f / DLS;
                            const int l = l0 + f % DLS;
                            __nv_bfloat16 *dst = p.Y + row * p.out_f + (long long)i * p.b * p.d + (long long)k * p.d + l;
                            *reinterpret_cast<uint4 *>(dst) =
                                *reinterpret_cast<const uint4 *>(stage + r * kEpiRowBytes + u * 16);
                        }
                    }
                    __syncwarp();
                }
                tc_fence_before();
                mbar_arrive(&acc_empty[buf]);
            }
        }
    }

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

struct TcLayout {
    int a_plane_bytes, v_stage_bytes, x_stage_bytes;
    int off_a, off_v, off_x, off_epi, off_bar, total;
};

TcLayout tc_layout(const Problem &p, int dls, int bk) {
    TcLayout L;
    auto up = [](int x) { return (x + 127) & ~127; };
    L.a_plane_bytes = (int)p.c * 256;               // 128 rows x c x 2 bytes
    L.v_stage_bytes = dls * bk * 32;               // dls planes x bk rows x 16 j x 2 bytes
    L.x_stage_bytes = 128 * kChunkJ * dls * 2;
    L.off_a = 0;
    L.off_v = up(L.off_a + dls * L.a_plane_bytes);
    L.off_x = up(L.off_v + kVStages * L.v_stage_bytes);
    L.off_epi = up(L.off_x + kXStages * L.x_stage_bytes);
    L.off_bar = L.off_epi + 4 * 32 * kEpiRowBytes;
    L.total = L.off_bar + (18 + kMaxSteps) * 8 + 16 + 128;  // + slack for base alignment
    return L;
}

}  // namespace

TcConfig tc_choose(const Problem &p) {
    const int dls = tc_dls(p);
    TcConfig c{dls, 0, kStepJ};
    if (!dls) return c;
    for (int bk = std::min<int>(256, 256 / dls); bk >= 16; bk -= 16)
        if (p.b % bk == 0) { c.bk = bk; break; }
    return c;
}

// k per epilogue chunk: a multiple of 16 dividing bk with dls * kc <= 128.
static int tc_kc(int dls, int bk) {
    for (int kc = std::min(bk, 128 / dls); kc >= 16; kc -= 16)
        if (bk % kc == 0) return kc;
    return 0;
}

bool tc_supported(const Problem &p, const char **why) {
    if (p.dtype != KS_BF16) { *why = "tensor-core kernel serves bf16"; return false; }
    const int dls = tc_dls(p);
    if (!dls) { *why = "d must be 1, 2, 4 or a multiple of 8"; return false; }
    if (p.c % kStepJ || p.c > 16 * kMaxSteps) { *why = "c must be a multiple of 16, at most 512"; return false; }
    if ((long long)p.c * dls > 512) { *why = "X slab (128 rows x c x DLS) exceeds the resident budget"; return false; }
    const uintptr_t al = reinterpret_cast<uintptr_t>(p.X) | reinterpret_cast<uintptr_t>(p.V) |
                         reinterpret_cast<uintptr_t>(p.Y);
    if (al % 16) { *why = "X, values and Y must be 16-byte aligned"; return false; }
    if (tc_choose(p).bk == 0) { *why = "no k-block size (multiple of 16, dividing b) fits"; return false; }
    if (p.batch > (1LL << 31) - 256) { *why = "batch too large for tensor-map coordinates"; return false; }
    return true;
}

template <int DLS>
static cudaError_t launch_dls(const Problem &pr, const TcConfig &cfg) {
    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap map;
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r;
    if (pr.d % 8 == 0) {
        cuuint64_t dims[4] = {(cuuint64_t)pr.d, (cuuint64_t)pr.c, (cuuint64_t)pr.a, (cuuint64_t)pr.batch};
        cuuint64_t strides[3] = {(cuuint64_t)pr.d * 2, (cuuint64_t)pr.c * pr.d * 2, (cuuint64_t)pr.in_features() * 2};
        cuuint32_t box[4] = {8, (cuuint32_t)kChunkJ, 1, (cuuint32_t)kRows};
        r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(pr.X), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        cuuint64_t dims[3] = {(cuuint64_t)(pr.c * pr.d), (cuuint64_t)pr.a, (cuuint64_t)pr.batch};
        cuuint64_t strides[2] = {(cuuint64_t)pr.c * pr.d * 2, (cuuint64_t)pr.in_features() * 2};
        cuuint32_t box[3] = {(cuuint32_t)(kChunkJ * pr.d), 1, (cuuint32_t)kRows};
        r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(pr.X), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

    const TcLayout L = tc_layout(pr, DLS, cfg.bk);
    TcParams p;
    p.V = static_cast<const __nv_bfloat16 *>(pr.V);
    p.Y = static_cast<__nv_bfloat16 *>(pr.Y);
    p.N = pr.batch;
    p.a = (int)pr.a; p.b = (int)pr.b; p.c = (int)pr.c; p.d = (int)pr.d;
    p.in_f = (int)pr.in_features();
    p.out_f = (int)pr.out_features();
    p.bk = cfg.bk;
    p.nkb = (int)(pr.b / cfg.bk);
    p.n_g = (int)(pr.a * (pr.d / DLS));
    p.kc = tc_kc(DLS, cfg.bk);
    if (p.kc == 0) return cudaErrorInvalidConfiguration;
    p.n_tiles = ((pr.batch + kRows - 1) / kRows) * p.n_g;
    p.status = device_status_ptr();
    if (!p.status) return cudaErrorUnknown;
    p.off_a = L.off_a; p.off_v = L.off_v; p.off_x = L.off_x; p.off_epi = L.off_epi; p.off_bar = L.off_bar;
    p.a_plane_bytes = L.a_plane_bytes;
    p.v_stage_bytes = L.v_stage_bytes;
    p.x_stage_bytes = L.x_stage_bytes;
    if (L.total > 232448) return cudaErrorInvalidConfiguration;
    auto kern = tc_kernel<DLS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (e != cudaSuccess) return e;
    const long long grid = std::min<long long>(p.n_tiles, (long long)sm_count());
    kern<<<(int)grid, kThreads, L.total, pr.stream>>>(map, p);
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
