// tcgen05 / TMEM / TMA kernels (filled in below the SIMT path).
#include "launch.h"

namespace gdn {

bool gdn_tc_supported(int, int) { return false; }
size_t gdn_tc_state_elems(int dk, int dv) { return (size_t)dk * dv; }
cudaError_t launch_gdn_tc(const GdnParams &, int, cudaStream_t) { return cudaErrorNotSupported; }
bool relu_tc_supported(int, int) { return false; }
cudaError_t launch_relu_tc(const ReluParams &, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace gdn
