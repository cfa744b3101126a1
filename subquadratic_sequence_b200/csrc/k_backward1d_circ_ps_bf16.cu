// 1-D backward pass in circular mode with a spectrum set per sample, bf16 activations.
#include "k_backward1d.cuh"

namespace hyena {
hyena_status_t dispatch_backward_circ_ps_bf16(int log2m, const Backward1dArgs& a, cudaStream_t st)
{
    return dispatch_backward<__nv_bfloat16, true, false>(log2m, a, st);
}
}  // namespace hyena
