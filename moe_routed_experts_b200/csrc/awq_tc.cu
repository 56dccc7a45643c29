// Grouped AWQ projections on tcgen05/TMEM tiles (large per-expert batches).
#include "proj.cuh"

namespace moe {

bool tc_available() { return false; }

moe_status launch_fwd_tc(const ProjParams &, int, bool, cudaStream_t) {
  return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "tcgen05 projection tiles are not built");
}

moe_status launch_bwd_tc(const BwdParams &, int, bool, cudaStream_t) {
  return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "tcgen05 projection tiles are not built");
}

}  // namespace moe
