// Four-step forward (L > 16384), bf16 activations.
#include "k_fourstep.cuh"

namespace hyena {
hyena_status_t dispatch_fourstep_bf16(int log2m, const FourStepArgs& a, int N, float2* scratch,
                                      cudaStream_t st)
{
    return dispatch_fourstep<__nv_bfloat16>(log2m, a, N, scratch, st);
}
}  // namespace hyena
