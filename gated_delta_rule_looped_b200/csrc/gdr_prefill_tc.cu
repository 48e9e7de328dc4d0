// gdr_prefill_tc.cu -- tensor-core (tcgen05 + TMA) chunked prefill.  Placeholder until the
// kernel lands: reports no supported shape, so every call takes the CUDA-core path.
#include "gdr_common.cuh"
#include "gdr_launch.h"

namespace lt2 {

bool prefill_tc_supports(int, int, int, int) { return false; }

cudaError_t launch_prefill_tc(const LoopSlice&, cudaStream_t, bool) { return cudaErrorNotSupported; }

}  // namespace lt2
