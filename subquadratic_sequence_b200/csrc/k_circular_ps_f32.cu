// Circular single-CTA forward with a spectrum set per sample, float32 activations.
#include "k_circular.cuh"

namespace hyena {
hyena_status_t dispatch_fused_circ_ps_f32(int log2m, const Fused1dArgs& a, cudaStream_t st)
{
    return dispatch_fused_circ<float, true>(log2m, a, st);
}
}  // namespace hyena
