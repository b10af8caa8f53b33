// The library's pattern heuristic: which kernel family runs a KS product.
//
// The KS-matmul abstract on the taxoreview.com page says a simple heuristic on
// the pattern parameters predicts when its fused kernel wins; its rule is not
// given, so this one is ours, chosen among our own kernels:
//
//   * tiny blocks (b*c <= 64, e.g. the 2x2 blocks of a butterfly): nothing to
//     reuse, so the streaming kernel, bound by HBM bandwidth;
//   * fp32: the CUDA-core gather-GEMM (the fp32 result must match fp32 FMA
//     arithmetic, so tensor cores are never chosen silently for KS_F32);
//   * TF32 / BF16 with b, c large enough that each (i, l) block is a real dense
//     GEMM (both >= 16 and multiples of the MMA granules): the tcgen05
//     tensor-core kernel; otherwise the gather-GEMM computing in fp32;
//   * anything the vector loaders cannot serve (odd d, unaligned pointers or
//     widths): the streaming kernel's scalar form.
#include "ks_internal.h"

namespace ks {

bool make_plan(const Problem &p, int variant, Plan *out, const char **why) {
    *why = "";
    Plan plan{};
    if (variant == KS_VARIANT_AUTO) {
        const char *w = "";
        if (p.b * p.c <= 64) {
            plan.variant = KS_VARIANT_STREAM;
        } else if (p.dtype != KS_F32 && tc_supported(p, &w)) {
            plan.variant = KS_VARIANT_TC;
        } else if (fma_supported(p, &w)) {
            plan.variant = KS_VARIANT_FMA;
        } else {
            plan.variant = KS_VARIANT_STREAM;
        }
    } else {
        plan.variant = variant;
        if (variant == KS_VARIANT_FMA && !fma_supported(p, why)) return false;
        if (variant == KS_VARIANT_TC && !tc_supported(p, why)) return false;
        if (variant == KS_VARIANT_STREAM && !stream_supported(p)) { *why = "stream"; return false; }
    }
    if (plan.variant == KS_VARIANT_FMA) plan.fma = fma_choose(p);
    if (plan.variant == KS_VARIANT_TC) plan.tc = tc_choose(p);
    *out = plan;
    return true;
}

}  // namespace ks
