// 3-D forward, bf16 activations.
#include "k_fft3d.cuh"

namespace hyena {
hyena_status_t dispatch_fft3d_bf16(int log2w, int log2h, int log2z, const Fft2dArgs& a, int N,
                                  float2* scratch, cudaStream_t st)
{
    return dispatch_fft3d<__nv_bfloat16>(log2w, log2h, log2z, a, N, scratch, st);
}
}  // namespace hyena
