// Single-CTA fused forward, bf16 activations.
#include "k_fused1d.cuh"

namespace hyena {
hyena_status_t dispatch_fused_bf16(int log2m, const Fused1dArgs& a, cudaStream_t st)
{
    return dispatch_fused<__nv_bfloat16>(log2m, a, st);
}
}  // namespace hyena
