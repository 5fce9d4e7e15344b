// tcgen05 mainloop (TMEM accumulators, TMA-staged K/V).  Not built yet:
// the launchers report SAGE_ERR_UNSUPPORTED and the library selects the
// mma.sync mainloop.
#include "sage_common.cuh"

namespace sage {
bool tc_available() { return false; }
int launch_attn_tc(const AttnParams&, cudaStream_t) { return SAGE_ERR_UNSUPPORTED; }
int launch_debug_qk_tc(const AttnParams&, int, int, int, int, int32_t*, cudaStream_t) {
  return SAGE_ERR_UNSUPPORTED;
}
}  // namespace sage
