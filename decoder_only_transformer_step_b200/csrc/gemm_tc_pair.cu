// Instantiations of the tcgen05 GEMM for the CTA-pair 256 x 256 tile, one per
// epilogue kind (compiled apart from the host code so the build runs them in
// parallel).
#include "gemm_tc.cuh"

namespace tcg {
TCG_FOR_EACH_KIND(TCG_INSTANTIATE, 256, true)
TCG_INSTANTIATE(256, true, EPI_CE_FWD)
}  // namespace tcg

// The pipeline-wait limit is a device variable of each compilation unit.
int gemm_tc_pair_set_wait_limit(unsigned long long ns) { return set_unit_wait_limit(ns); }
