// Four-step forward (L > 16384), float32 activations.
#include "k_fourstep.cuh"

namespace hyena {
hyena_status_t dispatch_fourstep_f32(int log2m, const FourStepArgs& a, int N, float2* scratch,
                                     cudaStream_t st)
{
    return dispatch_fourstep<float>(log2m, a, N, scratch, st);
}
}  // namespace hyena
