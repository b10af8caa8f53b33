// tcgen05 tensor-core block-GEMM for KS products in TF32 / BF16.
#include "ks_internal.h"

namespace ks {

bool tc_supported(const Problem &p, const char **why) {
    (void)p;
    *why = "tensor-core kernel not built yet";
    return false;
}

TcConfig tc_choose(const Problem &) { return TcConfig{0, 0, 0}; }

cudaError_t launch_tc(const Problem &, const TcConfig &) { return cudaErrorNotSupported; }

}  // namespace ks
