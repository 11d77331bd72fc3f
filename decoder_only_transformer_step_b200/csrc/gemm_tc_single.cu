// Instantiations of the tcgen05 GEMM for the single-CTA 128 x 256 and
// 128 x 128 tiles, one per epilogue kind.
#include "gemm_tc.cuh"

namespace tcg {
TCG_FOR_EACH_KIND(TCG_INSTANTIATE, 256, false)
TCG_INSTANTIATE(256, false, EPI_CE_FWD)
TCG_FOR_EACH_KIND(TCG_INSTANTIATE, 128, false)
}  // namespace tcg

// The pipeline-wait limit is a device variable of each compilation unit.
int gemm_tc_single_set_wait_limit(unsigned long long ns) { return set_unit_wait_limit(ns); }
