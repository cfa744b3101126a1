// Per-order forward with z spilled to HBM, float32 activations.
#include "k_spill.cuh"

namespace hyena {
hyena_status_t dispatch_order_f32(int log2m, const Fused1dOrderArgs& a, cudaStream_t st)
{
    return dispatch_order<float, float, float>(log2m, a, st);
}
}  // namespace hyena
