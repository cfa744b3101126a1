// Circular single-CTA forward with a spectrum set per sample, bf16 activations.
#include "k_circular.cuh"

namespace hyena {
hyena_status_t dispatch_fused_circ_ps_bf16(int log2m, const Fused1dArgs& a, cudaStream_t st)
{
    return dispatch_fused_circ<__nv_bfloat16, true>(log2m, a, st);
}
}  // namespace hyena
