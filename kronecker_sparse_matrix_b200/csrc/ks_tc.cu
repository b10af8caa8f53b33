// tcgen05 tensor-core block-GEMM for KS products: bf16 inputs (kind::f16) or
// fp32 inputs multiplied at TF32 precision (kind::tf32), both accumulating in
// fp32 in tensor memory; Y is written in the input's storage type (bf16
// rounded to nearest even, or fp32).
//
// Y[n, i*b*d + k*d + l] = sum_{j<c} values[i, l, k, j] * X[n, i*c*d + j*d + l]
// (taxoreview.com page on Kronecker-sparse matrix multiplication, first
// abstract: a fused output-stationary kernel, no permutation passes).
//
// For one block i and offset l this is the dense GEMM
//     D_l[n, k] = sum_j A_l[n, j] * B_l[k, j],  A_l = X[:, i, :, l],  B_l = values[i, l]
// with M = 128 rows of the batch, N = the k of one pass, K = c.
//
// A tile is 128 rows x one block i x DLS consecutive l (DLS = 16 for bf16
// when d % 16 == 0, DLS = 8 when d % 8 == 0, else DLS = d).  Its outputs for all l and all k of a pass (DLS * bp <=
// 512 fp32 columns) accumulate in tensor memory while X streams through a
// ring of 16/32 KB chunks exactly once per pass; most patterns need a single
// pass, so X is read once and Y written once.  Each pass is its own tile, and
// the passes of one X tile are consecutive tiles, which run at the same time on
// neighbouring CTAs and share X through L2.
//
// The two element types share every byte count: a chunk holds half as many j
// in fp32 as in bf16, so raw rows, values rows (and their swizzles), K steps
// (32 bytes: 16 bf16 or 8 fp32 per MMA) and the staging boxes are the same
// sizes; only the operand planes' core matrices (8 j lines x 16 bytes, i.e.
// 8 rows in bf16 and 4 rows in fp32), the MMA kind and the output packing
// differ.
//
//   warp 0      TMA producer: raw X chunks (128 rows x 128 or 256 bytes of
//               (j, l) elements; l innermost, the only shape a tensor map can
//               fetch from the strided layout) into the ring, and the values
//               of the same j range into a 3..4-deep ring, as DLS K-major
//               planes whose rows (one k, the chunk's j) carry the swizzle of
//               their width (a TMA copy moves about one box row per clock, so
//               the rows are made as wide as the chunk allows);
//   warps 2..5  (DLS > 1) transpose each chunk in place, in registers, from
//               [row][j][l] to one MN-major no-swizzle operand plane per l,
//               padded (and, for bf16, skewed) so that every quarter-warp's
//               16-byte accesses reach eight bank groups (for DLS = 16 each
//               warp transposes whole 8-row groups within their own 4 KB,
//               unpadded); for d = 1 the TMA box
//               already lands as the 128-byte-swizzled K-major tile the MMA
//               reads, and these warps idle;
//   warp 1      one thread issues tcgen05.mma (M=128, N=bp, K=32 bytes) per
//               plane and K step, commits to mbarriers;
//   warps 6..9  tcgen05.ld the accumulators (each warp its 32 TMEM lanes =
//               rows), convert to the storage type, interleave the l planes
//               back into Y's (k, l) order in a shared-memory staging box of 32
//               rows, and hand it to a TMA tensor store when the box is
//               contiguous in Y (d == DLS); for 32-byte l runs (fp32
//               with DLS = 8, bf16 with DLS = 16) and d > DLS, to a 4-D
//               tensor store whose box is [k][row][l] (32-byte runs of Y);
//               otherwise copy it out in 16-byte stores.
//
// TF32: the tensor core reads each fp32 operand at TF32 precision (10
// explicit mantissa bits); products and sums are fp32.
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
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "ks_epilogue.cuh"
#include "ks_internal.h"
#include "ks_sm100.cuh"

namespace ks {
namespace {

using namespace sm100;

constexpr int kRows = 128;         // MMA M
constexpr int kVStages = 4;        // values ring depth bound
constexpr int kMaxStages = 8;      // X ring depth bound
constexpr int kThreads = 320;      // 10 warps
constexpr int kLoadWarp0 = 2;      // warps 2..5
constexpr int kEpiWarp0 = 6;       // warps 6..9
constexpr int kEpiWarpBytes = 4096; // staging per epilogue warp: one box of 32 rows x 128 B
constexpr int kChunkBytes = 128;    // output bytes per row per epilogue chunk
constexpr int kBiasBytes = 2048;    // fused bias of one tile (bp * DLS * ES <= 2 KB), per buffer and warp
constexpr int kSmemLimit = 232448; // per-block opt-in maximum on sm_100

// j per MMA (K = 32 bytes): 16 bf16, 8 fp32 (TF32)
__host__ __device__ constexpr int step_j(int es) { return 32 / es; }
// j per X chunk: raw rows of 256 bytes for DLS = 8, 128 bytes for DLS < 8;
// DLS = 16 (bf16 only) takes one K step, 16 j x 16 l = 512-byte rows
__host__ __device__ constexpr int chunk_j(int dls, int es) {
    return dls == 16 ? 16 : (dls == 8 ? 32 : 128 / dls) / es;
}
__host__ __device__ constexpr int chunk_bytes(int dls, int es) { return kRows * chunk_j(dls, es) * dls * es; }
// Transposed operand planes (DLS > 1), one per l.
//   bf16: MN-major, no swizzle: core matrices of 8 j lines x 16 bytes (8
//         rows), 128 bytes each; the 16 row groups of a j octet 144 bytes
//         apart (one 16-byte pad each) so that the transposer's 16-byte stores
//         from one warp spread over all eight bank groups; j octets 16 * 144
//         bytes apart.
//   fp32: K-major with the 32-byte swizzle: one 32-byte row of 8 j (one TF32
//         K step) per batch row, 128 rows = 4 KB per j octet (the tensor
//         cores read TF32 operands K-major; the layout is the one the values
//         operand uses for rows of 32 bytes).
//   bf16 with DLS = 16: the planes of the 8 rows of a row group take the
//         4 KB the group's raw rows took (core matrix (l, j octet) at
//         (2 l + octet) * 128 bytes), so each group is transposed in place by
//         one warp, without padding: its lanes' units are chosen so that
//         every quarter-warp reaches eight bank groups in both directions.
__host__ __device__ constexpr int group_stride(int es) { return es == 2 ? 144 : 256; }
__host__ __device__ constexpr int octet_stride(int es) { return es == 2 ? 16 * 144 : 128 * 32; }
__host__ __device__ constexpr int plane_stride(int dls, int es) { return (chunk_j(dls, es) / 8) * octet_stride(es); }
// ring slot: the raw chunk, transposed in place into padded planes, rounded
// up to 1 KiB so that every slot (a TMA destination) and the values ring
// after the X ring keep the 1 KiB alignment of the ring's base (the largest
// swizzle atom: 8 rows x 128 bytes)
__host__ __device__ constexpr int slot_bytes(int dls, int es) {
    return (dls == 1 || dls == 16 ? chunk_bytes(dls, es) : dls * plane_stride(dls, es) + 1023) / 1024 * 1024;
}
// DLS = 16 planes: bytes between row groups (8 raw rows of 512 bytes)
constexpr int kG16 = 4096;
// The values of one chunk land as DLS planes of bp rows (k) x chunk_j j,
// K-major with the swizzle as wide as a row (chunk_j * es bytes): tcgen05
// layout type and the TMA swizzle mode for that width.
__host__ __device__ constexpr int v_row_bytes(int dls, int es) { return chunk_j(dls, es) * es; }
__host__ __device__ constexpr uint32_t v_layout(int dls, int es) {
    return v_row_bytes(dls, es) == 128 ? 2u : v_row_bytes(dls, es) == 64 ? 4u : 6u;
}

struct TcParams {
    const void *bias;  // fused epilogue: out_f values of the storage type, or null
    int act;
    long long N;
    int a, b, c, d;
    int out_f;
    int bp, passes, n_g, kc, nbuf;
    long long n_tiles;
    void *Y;
    unsigned *status;
    unsigned long long wait_ns;      // bound of the pipeline's mbarrier waits
    int stages;                      // X ring depth
    int vstages;                     // values ring depth
    int off_v, off_epi, off_bar;     // shared-memory carve-up (ring at offset 0)
    int v_stage_bytes;
    int box_elems, box_sw128;        // epilogue staging box: elements per row, swizzled
    int box_row_bytes;               // staging row stride when not swizzled (an odd number of 16-byte units)
    int ytma;                        // the staging box goes to Y as one TMA store: 2-D (d == DLS) or,
                                     // in the Y4 kernels, 4-D ([k][row][l] box, DLS * ES = 32, d > DLS)
    int x3d;                         // X chunks come from the (c*d, a, N) map (DLS < 8, or d == 8)
};

// Element type T: __nv_bfloat16 (kind::f16) or float (kind::tf32).
template <typename T>
__device__ __forceinline__ void mma_kind(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    if constexpr (sizeof(T) == 2)
        mma_bf16(d_tmem, adesc, bdesc, idesc, accumulate);
    else
        mma_tf32(d_tmem, adesc, bdesc, idesc, accumulate);
}

// 16-byte global -> shared copy (L2 only), its commit and the wait for all of
// this thread's copies.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// 4x4 transpose of 32-bit elements: in[r] holds elements e=0..3 of row r;
// out[e] holds rows r=0..3 of element e (a renaming of registers).
__device__ __forceinline__ void transpose4x4_b32(const uint4 (&in)[4], uint4 (&out)[4]) {
    out[0] = make_uint4(in[0].x, in[1].x, in[2].x, in[3].x);
    out[1] = make_uint4(in[0].y, in[1].y, in[2].y, in[3].y);
    out[2] = make_uint4(in[0].z, in[1].z, in[2].z, in[3].z);
    out[3] = make_uint4(in[0].w, in[1].w, in[2].w, in[3].w);
}

// EP: fused bias / activation epilogue compiled in; Y4: the output boxes go to
// a 4-D TMA store of [k][row][l] boxes (32-byte l runs, d > DLS), chosen at compile
// time so that the other instantiations carry none of it (a run-time choice
// cost the d == DLS TF32 epilogue 5-7%).
template <int DLS, typename T, bool EP, bool Y4 = false>
__global__ void __launch_bounds__(kThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap vmap,
              const __grid_constant__ CUtensorMap ymap, const TcParams p) {
    constexpr int ES = (int)sizeof(T);
    constexpr int KJ = step_j(ES);          // j per MMA
    constexpr int CTJ = chunk_j(DLS, ES);
    constexpr int CB = chunk_bytes(DLS, ES);
    constexpr int SB = slot_bytes(DLS, ES);
    constexpr int GS = group_stride(ES);
    constexpr int OS = octet_stride(ES);
    constexpr int PS = plane_stride(DLS, ES);
    constexpr int RPU = 16 / ES;            // rows of a core-matrix line (elements per 16-byte unit)
    constexpr int UNITS = CTJ * DLS * ES / 16;  // 16-byte units per raw row of a chunk (8 or 16)
    // bf16 transpose tasks (8 rows x one unit) per loader thread: 1 or 2
    constexpr int TASKS = (kRows / 8) * UNITS / 128;
    constexpr int CE = kChunkBytes / ES;    // output elements per staging row
    constexpr int KCM = CE / DLS;           // k per epilogue chunk, at most
    constexpr int LW = KCM < 8 ? KCM : 8;   // TMEM columns per load
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
    const int n_steps = p.c / KJ;
    const int n_chunks = (p.c + CTJ - 1) / CTJ;
    const int groups_per_i = p.d / DLS;
    const int S = p.stages;
    const int VS = p.vstages;
    const uint64_t wait_ns = p.wait_ns;

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
                for (int ch = 0; ch < n_chunks && ok; ++ch) {
                    const int xs = xq % S;
                    ok = mbar_wait(&x_empty[xs], ((xq / S) & 1) ^ 1, abort_flag, p.status, wait_ns);
                    if (!ok) break;
                    mbar_expect_tx(&x_full[xs], (uint32_t)CB);
                    if (DLS >= 8 && !p.x3d)
                        tma_load_4d(sR + xs * SB, &xmap, &x_full[xs], l0, ch * CTJ, i, n0);
                    else
                        tma_load_3d(sR + xs * SB, &xmap, &x_full[xs], ch * CTJ * p.d, i, n0);
                    ++xq;  // counted as soon as it is in flight (the abort drain relies on it)
                    // the values of the same CTJ j: values[i, l0:l0+DLS, pass k's, chunk j's]
                    const int vs = vq % VS;
                    ok = mbar_wait(&v_empty[vs], ((vq / VS) & 1) ^ 1, abort_flag, p.status, wait_ns);
                    if (!ok) break;
                    mbar_expect_tx(&v_full[vs], (uint32_t)p.v_stage_bytes);
                    tma_load_3d(sV + vs * p.v_stage_bytes, &vmap, &v_full[vs], ch * CTJ, ps * p.bp, i * p.d + l0);
                    ++vq;
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
            // D fp32 (bit 4); A and B bf16 (format 1, bits 7 and 10) or TF32
            // (format 2); A MN-major (bit 15) for bf16 with d > 1, K-major
            // otherwise; B K-major; N = bp (bits 17-22, N / 8), M = 128 (bits
            // 24-28, M / 16).
            const uint32_t fmt = (ES == 2) ? 1u : 2u;
            const uint32_t a_major = (DLS > 1 && ES == 2) ? 1u : 0u;
            const uint32_t idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | (a_major << 15) |
                                   ((uint32_t)(p.bp >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
            uint32_t xq = 0, vq = 0, accq = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++accq) {
                const int buf = (int)(accq % p.nbuf);
                ok = mbar_wait(&acc_empty[buf], ((accq / p.nbuf) & 1) ^ 1, abort_flag, p.status, wait_ns);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d_base = tmem_base + (uint32_t)(buf * DLS * p.bp);
                for (int ch = 0; ch < n_chunks && ok; ++ch, ++xq) {
                    const int xs = xq % S;
                    // d == 1: the TMA tile is the operand; otherwise wait for the transpose
                    ok = mbar_wait(DLS == 1 ? &x_full[xs] : &a_ready[xs], (xq / S) & 1, abort_flag, p.status,
                                   wait_ns);
                    if (!ok) break;
                    const int vs = vq % VS;
                    ok = mbar_wait(&v_full[vs], (vq / VS) & 1, abort_flag, p.status, wait_ns);
                    ++vq;
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t stage = su32(sR) + xs * SB;
                    const uint32_t vstage = su32(sV) + vs * p.v_stage_bytes;
                    for (int s = ch * CTJ / KJ; s < n_steps && s < (ch + 1) * CTJ / KJ; ++s) {
                        const int sl = s - ch * CTJ / KJ;  // K step within the chunk
#pragma unroll
                        for (int l = 0; l < DLS; ++l) {
                            uint64_t ad;
                            if (DLS == 1)
                                ad = smem_desc_sw128(stage + sl * 32, 1024);
                            else if (DLS == 16)  // MN-major, group-local planes: one K step per chunk
                                ad = smem_desc(stage + l * 256, 128, kG16);
                            else if (ES == 2)  // MN-major: a K step spans two j octets of the plane
                                ad = smem_desc(stage + l * PS + sl * 2 * OS, OS, GS);
                            else  // K-major, 32-byte swizzle: a K step is one j octet, 8-row atoms 256 bytes apart
                                ad = smem_desc_sw(stage + l * PS + sl * OS, GS, 6u);
                            // values stage: [l][bp k][CTJ j] swizzled rows, K step = 32 bytes
                            const uint32_t b_addr = vstage + l * (p.bp * CTJ * ES) + sl * 32;
                            const uint64_t bd = smem_desc_sw(b_addr, 8 * CTJ * ES, v_layout(DLS, ES));
                            mma_kind<T>(d_base + l * p.bp, ad, bd, idesc, s > 0 ? 1u : 0u);
                        }
                    }
                    mma_commit(&v_empty[vs]);
                    mma_commit(&x_empty[xs]);
                }
                if (ok) mma_commit(&acc_full[buf]);
            }
            // every MMA this thread issued has finished before TMEM is freed
            mma_commit(mma_done);
            mbar_wait_drain(mma_done, 0);
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------ in-place transpose (DLS > 1)
        if constexpr (DLS == 16) {
            // bf16, 16 l: raw row = 32 units of 16 bytes, unit q = (j = q / 2,
            // l half q % 2).  Warp tw takes row groups tw, tw + 4, tw + 8, tw + 12;
            // per group each lane reads one unit of the 8 rows, transposes it
            // and, after the whole warp has read, writes 8 lines (row group g,
            // l = 8 h + e, j) of the planes into the same 4 KB.  Lanes of a
            // quarter-warp take j = 0..7 (+8) with the l half flipped for the
            // upper four, so their reads (bank group q % 8) and their writes
            // (bank group j % 8) reach eight bank groups each.
            const int tw = warp - kLoadWarp0;  // 0..3
            const int quarter = lane >> 3, idx = lane & 7;
            const int h = (idx >> 2) ^ (quarter & 1);
            const int j = 8 * (quarter >> 1) + idx;
            const int q = 2 * j + h;
            uint32_t xq = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
                for (int ch = 0; ch < n_chunks; ++ch, ++xq) {
                    const int xs = xq % S;
                    const bool w = mbar_wait(&x_full[xs], (xq / S) & 1, abort_flag, p.status, wait_ns);
                    ok = bar_and(1, 128, w);  // uniform over the four loader warps
                    if (!ok) break;
                    uint8_t *st = sR + xs * SB;
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        uint8_t *gb = st + (4 * it + tw) * kG16;
                        uint4 in[8], out[8];
#pragma unroll
                        for (int r = 0; r < 8; ++r) in[r] = *reinterpret_cast<const uint4 *>(gb + r * 512 + q * 16);
                        transpose8x8_b16(in, out);
                        __syncwarp();  // every lane has read the group
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            *reinterpret_cast<uint4 *>(gb + (2 * (8 * h + e) + (j >> 3)) * 128 + (j & 7) * 16) = out[e];
                    }
                    fence_proxy_async();
                    mbar_arrive(&a_ready[xs]);
                }
            }
        } else if (DLS > 1 && ES == 2) {
            const int t = threadIdx.x - kLoadWarp0 * 32;  // 0..127
            // task -> (16-byte unit q of a raw row, group g of 8 rows).  16-byte
            // shared accesses are served eight lanes at a time, so every eight
            // consecutive lanes must reach eight distinct bank groups, both when
            // reading the raw chunk (group = q) and when writing the planes
            // (group = g + the unit's j mod 8, 144-byte row groups); for two and
            // four l the row group is skewed by the unit for that.
            auto task_unit = [&](int task, int &q, int &g) {
                if (DLS == 8) {
                    q = task % UNITS;
                    g = task / UNITS;
                } else {
                    q = task & 7;
                    g = ((task >> 3) + (q >> (DLS == 2 ? 1 : 2))) & 15;
                }
            };
            uint32_t xq = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
                for (int ch = 0; ch < n_chunks; ++ch, ++xq) {
                    const int xs = xq % S;
                    const bool w = mbar_wait(&x_full[xs], (xq / S) & 1, abort_flag, p.status, wait_ns);
                    ok = bar_and(1, 128, w);  // uniform over the four loader warps
                    if (!ok) break;
                    uint8_t *st = sR + xs * SB;
                    uint4 out[TASKS][8];
#pragma unroll
                    for (int k = 0; k < TASKS; ++k) {
                        int q, g;
                        task_unit(t + 128 * k, q, g);
                        uint4 in[8];
#pragma unroll
                        for (int r = 0; r < 8; ++r)
                            in[r] = *reinterpret_cast<const uint4 *>(st + ((g * 8 + r) * UNITS + q) * 16);
                        transpose8x8_b16(in, out[k]);
                    }
                    bar_sync(1, 128);  // every read of the raw chunk is done
#pragma unroll
                    for (int k = 0; k < TASKS; ++k) {
                        int q, g;
                        task_unit(t + 128 * k, q, g);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int f = 8 * q + e;
                            const int j = f / DLS, l = f % DLS;  // j within the chunk
                            *reinterpret_cast<uint4 *>(st + l * PS + (j >> 3) * OS + g * GS + (j & 7) * 16) =
                                out[k][e];
                        }
                    }
                    fence_proxy_async();
                    mbar_arrive(&a_ready[xs]);
                }
            }
        } else if (DLS > 1) {
            // fp32: per l a K-major plane of 32-byte rows (8 j) with the 32-byte
            // swizzle (16-byte half h of row n at h ^ bit 2 of n).  A task is one
            // batch row n and four consecutive j (a j quad jq) and, for DLS = 8,
            // four consecutive l (an l quad lq): 4x4 elements, read as four raw
            // units and written as four plane units (two for DLS = 2, whose raw
            // units hold 2 j x 2 l).  Consecutive lanes take lq, then jq, then n;
            // each lane starts its reads at a j rotated by its lane so that eight
            // lanes reach eight bank groups, and rotates the words back.
            constexpr int JQ = CTJ / 4;              // j quads per chunk: 2 (DLS 8, 4) or 4 (DLS 2)
            constexpr int LQ = DLS == 8 ? 2 : 1;     // l quads
            constexpr int TPR = JQ * LQ;             // tasks per row, = tasks per thread (128 rows)
            const int t = threadIdx.x - kLoadWarp0 * 32;  // 0..127
            uint32_t xq = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
                for (int ch = 0; ch < n_chunks; ++ch, ++xq) {
                    const int xs = xq % S;
                    const bool w = mbar_wait(&x_full[xs], (xq / S) & 1, abort_flag, p.status, wait_ns);
                    ok = bar_and(1, 128, w);  // uniform over the four loader warps
                    if (!ok) break;
                    uint8_t *st = sR + xs * SB;
                    uint4 out[TPR][4];
#pragma unroll
                    for (int k = 0; k < TPR; ++k) {
                        const int task = t + 128 * k;
                        const int lq = task % LQ, jq = (task / LQ) % JQ, n = task / TPR;
                        const uint8_t *row = st + n * (CTJ * DLS * 4);
                        if constexpr (DLS == 2) {
                            // raw units 2jq, 2jq+1 = (j 4jq..4jq+1, l 0..1), (j 4jq+2..4jq+3, l 0..1)
                            const int sw = n & 1;
                            const uint4 a0 = *reinterpret_cast<const uint4 *>(row + (2 * jq + sw) * 16);
                            const uint4 a1 = *reinterpret_cast<const uint4 *>(row + (2 * jq + 1 - sw) * 16);
                            const uint4 u0 = sw ? a1 : a0, u1 = sw ? a0 : a1;
                            out[k][0] = make_uint4(u0.x, u0.z, u1.x, u1.z);  // l = 0, j 4jq..4jq+3
                            out[k][1] = make_uint4(u0.y, u0.w, u1.y, u1.w);  // l = 1
                        } else {
                            // in[i] = raw unit of j = 4jq + ((i + rot) & 3), l = 4lq..4lq+3
                            const int rot = DLS == 8 ? ((jq + 2 * (n & 1)) & 3) : (n & 3);
                            uint4 in[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int j = 4 * jq + ((i + rot) & 3);
                                in[i] = *reinterpret_cast<const uint4 *>(row + (j * (DLS / 4) + lq) * 16);
                            }
                            uint4 o[4];
                            transpose4x4_b32(in, o);  // o[e] word i: l = 4lq + e, j = 4jq + ((i + rot) & 3)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                // word w must hold j = 4jq + w: rotate the words back by rot
                                uint4 v = o[e];
                                if (rot & 1) v = make_uint4(v.w, v.x, v.y, v.z);
                                if (rot & 2) v = make_uint4(v.z, v.w, v.x, v.y);
                                out[k][e] = v;
                            }
                        }
                    }
                    bar_sync(1, 128);  // every read of the raw chunk is done
#pragma unroll
                    for (int k = 0; k < TPR; ++k) {
                        const int task = t + 128 * k;
                        const int lq = task % LQ, jq = (task / LQ) % JQ, n = task / TPR;
                        const int half = (jq & 1) ^ ((n >> 2) & 1);  // the 32-byte swizzle
                        uint8_t *dst = st + (jq >> 1) * OS + n * 32 + half * 16;
#pragma unroll
                        for (int e = 0; e < (DLS == 2 ? 2 : 4); ++e)
                            *reinterpret_cast<uint4 *>(dst + (4 * lq + e) * PS) = out[k][e];
                    }
                    fence_proxy_async();
                    mbar_arrive(&a_ready[xs]);
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue: TMEM -> T -> Y
        // Per output chunk (kc k's, DLS*kc*ES <= 128 bytes per row): tcgen05.ld
        // the warp's 32 rows, convert in (k, l) order, write the rows into a
        // staging box (128-byte rows with the 16-byte units XOR-swizzled by row
        // when the row is full: conflict-free 16-byte stores and loads), then
        // copy the box to Y, four full 128-byte row segments per warp
        // instruction.
        const int ew = warp - kEpiWarp0;          // 0..3
        const int quad = warp & 3;                // TMEM lanes 32*quad .. 32*quad+31
        uint8_t *stage = sE + ew * kEpiWarpBytes; // 1024-aligned
        const int kc = p.kc;                      // k per chunk
        const int n_oc = p.bp / kc;
        const int units = DLS * kc * ES / 16;     // 16-byte output units per row per chunk
        const bool sw = p.box_sw128 != 0;
        // staging row stride (not sw): dense rows for the tensor store, else padded rows
        const int rsb = p.ytma ? p.box_elems * ES : p.box_row_bytes;
        const T *bias = static_cast<const T *>(p.bias);
        // Fused bias, DLS >= 4: the tile's bp x DLS columns, 16-byte units in
        // (k, l) order, go with cp.async to one of two buffers of this warp while
        // the warp drains the previous tile, so no chunk waits for a global load
        // (and no warp waits for another).  With DLS <= 2 a chunk's bias is one
        // contiguous 128-byte line that the chunk reads from L1 directly, which
        // measured faster there (d = 1, 2: 0.86-0.95x with the copies).
        constexpr bool kBiasSmem = DLS >= 4;
        uint8_t *sB = sE + 4 * kEpiWarpBytes + ew * 2 * kBiasBytes;
        auto bias_prefetch = [&](long long tile, int slot) {
            const int ps = (int)(tile % p.passes);
            const int g = (int)((tile / p.passes) % p.n_g);
            const int i = g / groups_per_i, l0 = (g % groups_per_i) * DLS;
            const int nu = p.bp * DLS / RPU;  // at most 128
            for (int U = lane; U < nu; U += 32) {
                const int f = RPU * U;  // first (k, l) element of the unit
                const T *src = bias + (long long)i * p.b * p.d + l0 + (long long)(ps * p.bp + f / DLS) * p.d + f % DLS;
                cp_async16(su32(sB) + slot * kBiasBytes + U * 16, src);
            }
            cp_async_commit();
        };
        if (EP && kBiasSmem && bias && blockIdx.x < p.n_tiles) bias_prefetch(blockIdx.x, 0);
        uint32_t accq = 0;
        bool ok = true;
        for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++accq) {
            const int ps = (int)(tile % p.passes);
            const long long t2 = tile / p.passes;
            const int g = (int)(t2 % p.n_g);
            const long long rb = t2 / p.n_g;
            const int i = g / groups_per_i, l0 = (g % groups_per_i) * DLS;
            const int row0 = (int)(rb * kRows) + 32 * quad;
            const int buf = (int)(accq % p.nbuf);
            ok = mbar_wait(&acc_full[buf], (accq / p.nbuf) & 1, abort_flag, p.status, wait_ns);
            ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
            if (EP && kBiasSmem && bias) {
                // this tile's bias has landed (every lane's copies, shown to the warp
                // by the sync); the other buffer, last read for the previous tile,
                // takes the next tile's
                cp_async_wait_all();
                __syncwarp();
                if (ok && tile + gridDim.x < p.n_tiles) bias_prefetch(tile + gridDim.x, (accq + 1) & 1);
            }
            if (!ok) break;
            const uint8_t *bias_tile = sB + (accq & 1) * kBiasBytes;
            tc_fence_after();
            for (int oc = 0; oc < n_oc; ++oc) {
                float acc[DLS][KCM];
                // bf16 with 1, 2 or 4 l: one load of the chunk's KCM columns per l plane
                // when they are whole (measured 1.03-1.05x on those patterns; TF32 kept the
                // narrow loads, 0.98-1.01x)
                constexpr bool kWide = ES == 2 && (KCM == 64 || KCM == 32 || KCM == 16);
                if (kWide && kc == KCM && p.bp % KCM == 0) {  // every column offset a multiple of the width
#pragma unroll
                    for (int l = 0; l < DLS; ++l) {
                        const uint32_t ta = tmem_base + ((uint32_t)(32 * quad) << 16) +
                                            (uint32_t)(buf * DLS * p.bp + l * p.bp + oc * kc);
                        if constexpr (KCM == 64) tmem_ld64(ta, acc[l]);
                        else if constexpr (KCM == 32) tmem_ld32(ta, acc[l]);
                        else if constexpr (KCM == 16) tmem_ld16(ta, acc[l]);
                    }
                } else {
#pragma unroll
                    for (int l = 0; l < DLS; ++l) {
#pragma unroll
                        for (int pc = 0; pc < KCM / LW; ++pc) {
                            if (pc * LW < kc) {
                                const uint32_t col = (uint32_t)(buf * DLS * p.bp + l * p.bp + oc * kc + pc * LW);
                                const uint32_t ta = tmem_base + ((uint32_t)(32 * quad) << 16) + col;
                                if constexpr (LW == 8) {
                                    float v[8];
                                    tmem_ld8(ta, v);
#pragma unroll
                                    for (int qq = 0; qq < 8; ++qq) acc[l][pc * 8 + qq] = v[qq];
                                } else {
                                    float v[4];
                                    tmem_ld4(ta, v);
#pragma unroll
                                    for (int qq = 0; qq < 4; ++qq) acc[l][pc * 4 + qq] = v[qq];
                                }
                            }
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
                if (EP && bias) {
                    // fused epilogue on (k = kq + e, l): the chunk's bias, units oc * units + u
                    // of the tile's copy, or 16-byte units of RPU consecutive (k, l) read
                    // directly (either way the same address for every lane: a broadcast)
#pragma unroll
                    for (int u = 0; u < CE / RPU; ++u) {
                        if (u < units) {
                            uint4 w;
                            if constexpr (kBiasSmem) {
                                w = *reinterpret_cast<const uint4 *>(bias_tile + (oc * units + u) * 16);
                            } else {
                                const int e0 = (RPU * u) / DLS, lu = (RPU * u) % DLS;
                                w = __ldg(reinterpret_cast<const uint4 *>(bias + ybase + (long long)(kq + e0) * p.d + lu));
                            }
                            float bb[RPU];
                            if constexpr (ES == 2) {
                                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                                for (int h = 0; h < 4; ++h) {
                                    const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ww[h]));
                                    bb[2 * h] = f2.x;
                                    bb[2 * h + 1] = f2.y;
                                }
                            } else {
                                bb[0] = __uint_as_float(w.x);
                                bb[1] = __uint_as_float(w.y);
                                bb[2] = __uint_as_float(w.z);
                                bb[3] = __uint_as_float(w.w);
                            }
#pragma unroll
                            for (int h = 0; h < RPU; ++h) {
                                const int f = RPU * u + h;
                                acc[f % DLS][f / DLS] += bb[h];
                            }
                        }
                    }
                }
                if (EP && p.act) {
                    if (p.act == 2) {
                        static_assert(KCM % 2 == 0, "pairs of columns");
                        // GELU, tanh form, two values per step in the packed fp32
                        // instructions: u = z (c0 + c1 z^2) with c0 = sqrt(2/pi) and
                        // c1 = 0.044715 c0, h = z / 2, h + h tanh(u) (the hardware
                        // tanh).  The whole chunk in one block, so the scheduler can
                        // interleave every element's chain: 1.23x on GPT-2 bf16 with
                        // bias + GELU against one element at a time; the same
                        // arithmetic split per l plane, or moved into a helper that
                        // takes the tile, measured 1.0x and 1.06x.
#pragma unroll
                        for (int l = 0; l < DLS; ++l) {
#pragma unroll
                            for (int e = 0; e + 1 < KCM; e += 2) {
                                const float2 z = make_float2(acc[l][e], acc[l][e + 1]);
                                const float2 z2 = __fmul2_rn(z, z);
                                const float2 q = __ffma2_rn(z2, make_float2(0.0356774081f, 0.0356774081f),
                                                            make_float2(0.7978845608f, 0.7978845608f));
                                const float2 u = __fmul2_rn(z, q);
                                const float2 h = __fmul2_rn(z, make_float2(0.5f, 0.5f));
                                const float2 t = make_float2(tanh_hw(u.x), tanh_hw(u.y));
                                const float2 y = __ffma2_rn(h, t, h);
                                acc[l][e] = y.x;
                                acc[l][e + 1] = y.y;
                            }
                        }
                    } else {
#pragma unroll
                        for (int l = 0; l < DLS; ++l) ep_act_array(acc[l], p.act);
                    }
                }
                if (p.ytma) {  // the previous box store has finished reading the staging
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
                }
                // unit u = elements RPU*u .. RPU*u+RPU-1 of (k*DLS + l)
#pragma unroll
                for (int u = 0; u < CE / RPU; ++u) {
                    if (u < units) {
                        uint32_t w[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            if constexpr (ES == 2) {
                                const int f0 = 8 * u + 2 * h, f1 = f0 + 1;
                                w[h] = pack_bf16x2(acc[f0 % DLS][f0 / DLS], acc[f1 % DLS][f1 / DLS]);
                            } else {
                                const int f = 4 * u + h;
                                w[h] = __float_as_uint(acc[f % DLS][f / DLS]);
                            }
                        }
                        uint32_t off = sw ? lane * 128 + ((u ^ (lane & 7)) << 4) : lane * rsb + u * 16;
                        // 4-D box (DLS * ES = 32): [k][row][l], unit u = (k, l0u .. l0u + RPU - 1); the
                        // eight lanes of a 16-byte store reach at least four bank groups
                        if constexpr (Y4)
                            off = ((RPU * u) / DLS) * (32 * DLS * ES) + lane * (DLS * ES) + ((RPU * u) % DLS) * ES;
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
                        if constexpr (Y4)
                            tma_store_4d(&ymap, su32(stage), l0, row0, kq, i);
                        else
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
                        const int f = RPU * u;
                        const long long col = ybase + (long long)(kq + f / DLS) * p.d + f % DLS;
                        int r = lane >> 3;
                        T *yp = static_cast<T *>(p.Y) + (long long)(row0 + r) * p.out_f + col;
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

// bf16 takes 16 l per tile where that measured faster than 8 on all 66 bf16
// sweep patterns with d >= 16 at 25088 rows: d a multiple of 64 with c <= 96
// (X boxes of 32-byte rows instead of 16; 1.05-1.17x), and d = 16 with b not a
// multiple of 32 (passes of 16 k with double-buffered accumulators; 1.02-1.15x).
// Elsewhere the passes of at most 32 k, which repeat the copy and transpose of
// every X chunk twice as often as 8 l with 64 k, made it 0.77-0.99x.
int tc_dls(const Problem &p) {
    if (p.dtype == KS_BF16 && p.d % 16 == 0 && ((p.d % 64 == 0 && p.c <= 96) || (p.d == 16 && p.b % 32 != 0)))
        return 16;
    if (p.d % 8 == 0) return 8;
    if (p.d == 1 || p.d == 2 || p.d == 4) return (int)p.d;
    return 0;
}

int tc_es(const Problem &p) { return p.dtype == KS_BF16 ? 2 : 4; }

// k per epilogue chunk: a multiple of the TMEM load width (8 columns, or 4
// when a 128-byte row holds fewer than 8 k) dividing bp with
// dls * kc * es <= 128 bytes, preferring rows of exactly 128 bytes (one
// swizzled store box).
int tc_kc(int dls, int bp, int es) {
    const int ce = kChunkBytes / es, kcm = ce / dls, lw = kcm < 8 ? kcm : 8;
    for (int kc = std::min(bp, kcm) / lw * lw; kc >= lw; kc -= lw)
        if (bp % kc == 0 && dls * kc == ce) return kc;
    for (int kc = std::min(bp, kcm) / lw * lw; kc >= lw; kc -= lw)
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
// staging (and, with a fused bias and DLS >= 4, two tiles of bias per epilogue
// warp), barriers.
bool tc_layout(int dls, int bp, int es, bool bias, TcLayout *out) {
    const bool ep = bias && dls >= 4;
    TcLayout L;
    auto up = [](int x, int a) { return (x + a - 1) / a * a; };
    const int cb = slot_bytes(dls, es);
    L.v_stage_bytes = es * bp * chunk_j(dls, es) * dls;
    if (bp * dls * es > kBiasBytes) return false;
    const int epi = 4 * kEpiWarpBytes + (ep ? 4 * 2 * kBiasBytes : 0);
    const int budget = kSmemLimit - 2048 - 4 * kEpiWarpBytes - kBarBytes;  // alignment slack
    auto x_stages = [&](int bud, int vs) {
        return std::min(kMaxStages, (bud - up(vs * L.v_stage_bytes, 128)) / cb);
    };
    L.vstages = (kVStages * L.v_stage_bytes + 3 * cb <= budget) ? kVStages : 3;
    L.stages = x_stages(budget, L.vstages);
    if (ep) {  // the bias buffers come out of a values stage rather than an X stage where possible
        const int bud = budget - 4 * 2 * kBiasBytes;
        int vs = L.vstages, st = x_stages(bud, vs);
        if (st < L.stages && vs == kVStages && x_stages(bud, 3) > st) st = x_stages(bud, vs = 3);
        L.vstages = vs;
        L.stages = st;
    }
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

// KS_FAULT_INJECT=timeout: the tensor-core pipelines' waits give up at once
// (tests of the device status word); otherwise about one second.
unsigned long long pipeline_wait_bound_ns() {
    const char *f = getenv("KS_FAULT_INJECT");
    return (f && strcmp(f, "timeout") == 0) ? 0ull : (unsigned long long)sm100::kTimeoutNs;
}

TcConfig tc_choose(const Problem &p) {
    const int dls = tc_dls(p);
    TcConfig c{dls, 0, step_j(tc_es(p))};
    if (dls) c.bk = tc_bp(dls, p.b);
    return c;
}

bool tc_supported(const Problem &p, const char **why) {
    if (p.dtype == KS_F32) {
        *why = "fp32 products keep fp32 arithmetic (CUDA cores); the tensor-core kernel serves KS_TF32 and KS_BF16";
        return false;
    }
    const int es = tc_es(p);
    const int dls = tc_dls(p);
    if (!dls) { *why = "d must be 1, 2, 4 or a multiple of 8"; return false; }
    if (p.c % step_j(es)) {
        *why = es == 2 ? "c must be a multiple of 16 (bf16)" : "c must be a multiple of 8 (TF32)";
        return false;
    }
    const uintptr_t al = reinterpret_cast<uintptr_t>(p.X) | reinterpret_cast<uintptr_t>(p.V) |
                         reinterpret_cast<uintptr_t>(p.Y);
    if (al % 16) { *why = "X, values and Y must be 16-byte aligned"; return false; }
    if (reinterpret_cast<uintptr_t>(p.bias) % 16) { *why = "a fused bias must be 16-byte aligned"; return false; }
    const int bp = tc_bp(dls, p.b);
    TcLayout L;
    if (bp == 0 || tc_kc(dls, bp, es) == 0) { *why = "b has no pass width (a multiple of 16 dividing it)"; return false; }
    if (!tc_layout(dls, bp, es, p.bias != nullptr, &L)) { *why = "shared memory budget"; return false; }
    if (p.batch > (1LL << 31) - 256 || p.a * p.d > (1LL << 31)) { *why = "sizes exceed tensor-map coordinates"; return false; }
    return true;
}

template <int DLS, typename T>
static cudaError_t launch_dls(const Problem &pr, const TcConfig &cfg) {
    constexpr int ES = (int)sizeof(T);
    constexpr CUtensorMapDataType kType = ES == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    const int bp = cfg.bk;
    TcLayout L;
    if (bp == 0 || !tc_layout(DLS, bp, ES, pr.bias != nullptr, &L)) return cudaErrorInvalidConfiguration;
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUtensorMap xmap, vmap;
    CUresult r;
    const bool x3d = DLS < 8 || pr.d == DLS;
    if (!x3d) {
        // X as (d, c, a, N): a box (DLS l, CTJ j, 1, 128 rows) = [row][j][l]
        cuuint64_t dims[4] = {(cuuint64_t)pr.d, (cuuint64_t)pr.c, (cuuint64_t)pr.a, (cuuint64_t)pr.batch};
        cuuint64_t strides[3] = {(cuuint64_t)pr.d * ES, (cuuint64_t)pr.c * pr.d * ES,
                                 (cuuint64_t)pr.in_features() * ES};
        cuuint32_t box[4] = {(cuuint32_t)DLS, (cuuint32_t)chunk_j(DLS, ES), 1, (cuuint32_t)kRows};
        r = encode(&xmap, kType, 4, const_cast<void *>(pr.X), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        // X as (c*d, a, N): a box (CTJ*DLS elements, 1, 128 rows) = [row][(j, l)]
        // (d == DLS: whole 256- or 512-byte rows for DLS = 8 or 16); for d == 1 with the
        // 128-byte swizzle, the K-major operand tile itself
        cuuint64_t dims[3] = {(cuuint64_t)(pr.c * pr.d), (cuuint64_t)pr.a, (cuuint64_t)pr.batch};
        cuuint64_t strides[2] = {(cuuint64_t)pr.c * pr.d * ES, (cuuint64_t)pr.in_features() * ES};
        cuuint32_t box[3] = {(cuuint32_t)(chunk_j(DLS, ES) * DLS), 1, (cuuint32_t)kRows};
        r = encode(&xmap, kType, 3, const_cast<void *>(pr.X), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   DLS == 1 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    {
        // values[i][l][k][j] viewed as (j, k, i*d+l): a box (CTJ j, bp k, DLS l)
        // lands as DLS planes [k][CTJ j], rows of CTJ*ES bytes swizzled at that
        // width: the K-major operand for CTJ*ES/32 K steps.  (A TMA fetches
        // about one box row per clock, so rows of 16 bytes would cap the copy
        // far below the bandwidth this kernel needs.)
        cuuint64_t dims[3] = {(cuuint64_t)pr.c, (cuuint64_t)pr.b, (cuuint64_t)(pr.a * pr.d)};
        cuuint64_t strides[2] = {(cuuint64_t)pr.c * ES, (cuuint64_t)pr.b * pr.c * ES};
        cuuint32_t box[3] = {(cuuint32_t)chunk_j(DLS, ES), (cuuint32_t)bp, (cuuint32_t)DLS};
        const int rb = v_row_bytes(DLS, ES);
        const CUtensorMapSwizzle vsw = rb == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                       : rb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : CU_TENSOR_MAP_SWIZZLE_32B;
        r = encode(&vmap, kType, 3, const_cast<void *>(pr.V), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   vsw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    // epilogue chunk: kc k's; rows of 128 bytes use the swizzled staging box
    const int kc = tc_kc(DLS, bp, ES);
    if (kc == 0) return cudaErrorInvalidConfiguration;
    const int bi = DLS * kc;  // elements per staging row
    const bool sw128 = bi * ES == kChunkBytes;
    const bool yal = (reinterpret_cast<uintptr_t>(pr.Y) % 16) == 0;
    const bool ytma = pr.d == DLS && yal;
    // 32-byte l runs (fp32 with DLS = 8, bf16 with DLS = 16) and d > DLS: Y
    // viewed as (d, N, b, a), a box (DLS l, 32 rows, kc k, 1 block) whose
    // shared image is [k][row][l] with 32-byte (k, row) runs and no swizzle.
    // (Measured against the 16-byte stores: 1.11x median on the d >= 16 TF32
    // patterns; for bf16 with DLS = 8 the 16-byte runs made it slower.)
    constexpr bool kY4 = DLS * ES == 32;
    const bool y4d = kY4 && pr.d > DLS && yal;
    CUtensorMap ymap;
    memset(&ymap, 0, sizeof(ymap));
    if (y4d) {
        cuuint64_t dims[4] = {(cuuint64_t)pr.d, (cuuint64_t)pr.batch, (cuuint64_t)pr.b, (cuuint64_t)pr.a};
        cuuint64_t strides[3] = {(cuuint64_t)pr.out_features() * ES, (cuuint64_t)pr.d * ES,
                                 (cuuint64_t)pr.b * pr.d * ES};
        cuuint32_t box[4] = {(cuuint32_t)DLS, 32, (cuuint32_t)kc, 1};
        r = encode(&ymap, kType, 4, pr.Y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    if (ytma) {
        // Y as (out_f, N): a box (DLS*kc elements, 32 rows); 128-byte rows with the
        // 128-byte swizzle of the staging, shorter rows packed densely
        cuuint64_t dims[2] = {(cuuint64_t)pr.out_features(), (cuuint64_t)pr.batch};
        cuuint64_t strides[1] = {(cuuint64_t)pr.out_features() * ES};
        cuuint32_t box[2] = {(cuuint32_t)bi, 32};
        r = encode(&ymap, kType, 2, pr.Y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }

    TcParams p;
    p.box_elems = bi;
    p.box_sw128 = sw128 ? 1 : 0;
    p.box_row_bytes = bi * ES + ((bi * ES / 16) % 2 == 0 ? 16 : 0);
    p.ytma = ytma ? 1 : y4d ? 2 : 0;
    p.x3d = x3d ? 1 : 0;
    p.N = pr.batch;
    p.bias = pr.bias;
    p.act = pr.act;
    p.a = (int)pr.a; p.b = (int)pr.b; p.c = (int)pr.c; p.d = (int)pr.d;
    p.out_f = (int)pr.out_features();
    p.bp = bp;
    p.passes = (int)(pr.b / bp);
    p.n_g = (int)(pr.a * (pr.d / DLS));
    p.kc = kc;
    p.nbuf = (2 * DLS * bp <= 512) ? 2 : 1;
    // tiles = (row block, l group, pass of k), the pass varying fastest: CTAs
    // that run side by side take the passes of the same X tile, so its second
    // read is served by L2
    p.n_tiles = ((pr.batch + kRows - 1) / kRows) * p.n_g * p.passes;
    p.Y = pr.Y;
    p.status = device_status_ptr();
    if (!p.status) return cudaErrorUnknown;
    p.wait_ns = pipeline_wait_bound_ns();
    p.stages = L.stages;
    p.vstages = L.vstages;
    p.off_v = L.off_v;
    p.off_epi = L.off_epi;
    p.off_bar = L.off_bar;
    p.v_stage_bytes = L.v_stage_bytes;
    const bool ep = pr.bias || pr.act;
    auto kern = ep ? tc_kernel<DLS, T, true> : tc_kernel<DLS, T, false>;
    if constexpr (kY4)
        if (y4d) kern = ep ? tc_kernel<DLS, T, true, true> : tc_kernel<DLS, T, false, true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (e != cudaSuccess) return e;
    const long long grid = std::min<long long>(p.n_tiles, (long long)sm_count());
    kern<<<(int)grid, kThreads, L.total, pr.stream>>>(xmap, vmap, ymap, p);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_typed(const Problem &p, const TcConfig &cfg) {
    switch (cfg.dl) {
        case 16:
            if constexpr (sizeof(T) == 2) return launch_dls<16, T>(p, cfg);
            return cudaErrorInvalidConfiguration;
        case 8: return launch_dls<8, T>(p, cfg);
        case 4: return launch_dls<4, T>(p, cfg);
        case 2: return launch_dls<2, T>(p, cfg);
        case 1: return launch_dls<1, T>(p, cfg);
        default: return cudaErrorInvalidConfiguration;
    }
}

void *tensor_map_encoder() { return reinterpret_cast<void *>(encode_fn()); }

cudaError_t launch_tc(const Problem &p, const TcConfig &cfg) {
    if (p.dtype == KS_BF16) return launch_typed<__nv_bfloat16>(p, cfg);
    if (p.dtype == KS_TF32) return launch_typed<float>(p, cfg);
    return cudaErrorInvalidValue;
}

}  // namespace ks
