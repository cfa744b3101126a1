// Circular 1-D forward, bf16 activations.
#include "k_circular.cuh"

namespace hyena {
hyena_status_t dispatch_fused_circ_bf16(int log2m, const Fused1dArgs& a, cudaStream_t st)
{
    return dispatch_fused_circ<__nv_bfloat16>(log2m, a, st);
}
}  // namespace hyena
