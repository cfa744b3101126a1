// 1-D backward pass in circular mode with a spectrum set per sample, float32 activations.
#include "k_backward1d.cuh"

namespace hyena {
hyena_status_t dispatch_backward_circ_ps_f32(int log2m, const Backward1dArgs& a, cudaStream_t st)
{
    return dispatch_backward<float, true, false>(log2m, a, st);
}
}  // namespace hyena
