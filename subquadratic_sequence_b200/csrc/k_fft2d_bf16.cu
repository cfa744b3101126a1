// 2-D forward with bf16 activations.
#include "k_fft2d.cuh"

namespace hyena {
hyena_status_t dispatch_fft2d_bf16(int log2w, int log2h, const Fft2dArgs& a, int N, float2* scratch,
                                   cudaStream_t st)
{
    return dispatch_fft2d<__nv_bfloat16>(log2w, log2h, a, N, scratch, st);
}
}  // namespace hyena
