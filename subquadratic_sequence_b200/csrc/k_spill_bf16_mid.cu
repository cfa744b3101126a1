// Per-order forward with z spilled to HBM, bf16 activations, middle orders (z float32).
#include "k_spill.cuh"

namespace hyena {
hyena_status_t dispatch_order_bf16_mid(int log2m, const Fused1dOrderArgs& a, cudaStream_t st)
{
    return dispatch_order<__nv_bfloat16, float, float>(log2m, a, st);
}
}  // namespace hyena
