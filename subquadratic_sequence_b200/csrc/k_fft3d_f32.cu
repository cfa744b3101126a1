// 3-D forward (padded and circular), float32 activations.
#include "k_fft3d.cuh"

namespace hyena {
// log2m: log2 of the slots per row (W padded, W/2 circular)
hyena_status_t dispatch_fft3d_f32(int log2m, int log2h, int log2z, const Fft2dArgs& a, int N,
                                  float2* scratch, cudaStream_t st, bool pad)
{
    return pad ? dispatch_fft3d<float, true>(log2m, log2h, log2z, a, N, scratch, st)
               : dispatch_fft3d<float, false>(log2m, log2h, log2z, a, N, scratch, st);
}
}  // namespace hyena
