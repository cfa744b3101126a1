// Four-step backward in circular mode (16384 < L <= 2^22), float32 activations.
#include "k_fourstep_bwd.cuh"

namespace hyena {
hyena_status_t dispatch_fourstep_bwd_circ_f32(int log2m, const FourStepBwdArgs& a, int N, cudaStream_t st)
{
    return dispatch_fourstep_bwd_circ<float>(log2m, a, N, st);
}
}  // namespace hyena
