// Single-CTA fused forward, float32 activations.
#include "k_fused1d.cuh"

namespace hyena {
hyena_status_t dispatch_fused_f32(int log2m, const Fused1dArgs& a, cudaStream_t st)
{
    return a.H_bstride ? dispatch_fused_ps_f32(log2m, a, st) : dispatch_fused<float, false>(log2m, a, st);
}
}  // namespace hyena
