// fwd_tc.cu -- tcgen05/TMEM tensor-core causal Polar Attention prefill (sm_100a).
#include "polar_common.cuh"
#include "polar_internal.h"

namespace polar {
cudaError_t launch_fwd_tc(const FwdLaunch &) { return cudaErrorNotSupported; }
}  // namespace polar
