// Per-order forward with z spilled to HBM, bf16 activations, first order (v bf16, z_1 float32).
#include "k_spill.cuh"

namespace hyena {
hyena_status_t dispatch_order_bf16_first(int log2m, const Fused1dOrderArgs& a, cudaStream_t st)
{
    return dispatch_order<__nv_bfloat16, __nv_bfloat16, float>(log2m, a, st);
}
}  // namespace hyena
