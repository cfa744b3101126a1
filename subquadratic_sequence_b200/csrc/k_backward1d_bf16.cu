// 1-D backward pass, bf16 activations.
#include "k_backward1d.cuh"

namespace hyena {
hyena_status_t dispatch_backward_bf16(int log2m, const Backward1dArgs& a, cudaStream_t st)
{
    return dispatch_backward<__nv_bfloat16>(log2m, a, st);
}
}  // namespace hyena
