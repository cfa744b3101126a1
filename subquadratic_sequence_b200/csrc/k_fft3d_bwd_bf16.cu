// 3-D backward (padded and circular), bf16 activations.
#include "k_fft3d_bwd.cuh"

namespace hyena {
hyena_status_t dispatch_bwd3d_bf16(int log2m, int log2h, int log2z, const Bwd2dArgs& a, int N, cudaStream_t st,
                                  bool pad)
{
    return dispatch_bwd3d<__nv_bfloat16>(log2m, log2h, log2z, a, N, st, pad);
}
}  // namespace hyena
