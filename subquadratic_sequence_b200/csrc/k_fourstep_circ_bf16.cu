// Four-step forward in circular mode (16384 < L <= 2^22), bf16 activations.
#include "k_fourstep.cuh"

namespace hyena {
hyena_status_t dispatch_fourstep_circ_bf16(int log2m, const FourStepArgs& a, int N, float2* scratch,
                                          cudaStream_t st)
{
    return dispatch_fourstep_circ<__nv_bfloat16>(log2m, a, N, scratch, st);
}
}  // namespace hyena
