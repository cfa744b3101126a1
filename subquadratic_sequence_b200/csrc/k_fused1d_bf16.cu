// Single-CTA fused forward, bf16 activations.
#include "k_fused1d.cuh"

namespace hyena {
hyena_status_t dispatch_fused_bf16(int log2m, const Fused1dArgs& a, cudaStream_t st)
{
    return a.H_bstride ? dispatch_fused_ps_bf16(log2m, a, st) : dispatch_fused<__nv_bfloat16, false>(log2m, a, st);
}
}  // namespace hyena
