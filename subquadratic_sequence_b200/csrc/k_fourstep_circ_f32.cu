// Four-step forward in circular mode (16384 < L <= 2^22), float32 activations.
#include "k_fourstep.cuh"

namespace hyena {
hyena_status_t dispatch_fourstep_circ_f32(int log2m, const FourStepArgs& a, int N, float2* scratch,
                                          cudaStream_t st)
{
    return dispatch_fourstep_circ<float>(log2m, a, N, scratch, st);
}
}  // namespace hyena
