// Circular 1-D forward, float32 activations.
#include "k_circular.cuh"

namespace hyena {
hyena_status_t dispatch_fused_circ_f32(int log2m, const Fused1dArgs& a, cudaStream_t st)
{
    return dispatch_fused_circ<float>(log2m, a, st);
}
}  // namespace hyena
