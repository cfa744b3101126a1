// Four-step backward in circular mode (16384 < L <= 2^22), bf16 activations.
#include "k_fourstep_bwd.cuh"

namespace hyena {
hyena_status_t dispatch_fourstep_bwd_circ_bf16(int log2m, const FourStepBwdArgs& a, int N, cudaStream_t st)
{
    return dispatch_fourstep_bwd_circ<__nv_bfloat16>(log2m, a, N, st);
}
}  // namespace hyena
