// 2-D backward, float32 activations.
#include "k_fft2d_bwd.cuh"

namespace hyena {
hyena_status_t dispatch_bwd2d_f32(int log2w, int log2h, const Bwd2dArgs& a, int N, cudaStream_t st)
{
    return dispatch_bwd2d<float>(log2w, log2h, a, N, st);
}
}  // namespace hyena
