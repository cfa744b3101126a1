// 2-D backward pass in circular mode, bf16 activations.
#include "k_fft2d_bwd.cuh"

namespace hyena {
hyena_status_t dispatch_bwd2d_circ_bf16(int log2m, int log2h, const Bwd2dArgs& a, int N, cudaStream_t st)
{
    return dispatch_bwd2d_circ<__nv_bfloat16>(log2m, log2h, a, N, st);
}
}  // namespace hyena
