// k_spill.cuh -- launchers of the per-order forward (z spilled to HBM between
// orders), included by one .cu file per combination of storage types.
#pragma once

#include "launch.cuh"

namespace hyena {

template <int LOG2M, typename IO, typename ZIN, typename ZOUT>
hyena_status_t launch_order(const Fused1dOrderArgs& a, cudaStream_t st)
{
    using F = Fft1d<LOG2M>;
    const long BD = (long)a.B * a.D;
    return launch(fused1d_order_kernel<LOG2M, IO, ZIN, ZOUT>, (unsigned)((BD + F::G - 1) / F::G), F::THREADS,
                  F::SMEM_BYTES, st, a);
}

template <typename IO, typename ZIN, typename ZOUT>
hyena_status_t dispatch_order(int log2m, const Fused1dOrderArgs& a, cudaStream_t st)
{
    switch (log2m) {
    case 4: return launch_order<4, IO, ZIN, ZOUT>(a, st);
    case 5: return launch_order<5, IO, ZIN, ZOUT>(a, st);
    case 6: return launch_order<6, IO, ZIN, ZOUT>(a, st);
    case 7: return launch_order<7, IO, ZIN, ZOUT>(a, st);
    case 8: return launch_order<8, IO, ZIN, ZOUT>(a, st);
    case 9: return launch_order<9, IO, ZIN, ZOUT>(a, st);
    case 10: return launch_order<10, IO, ZIN, ZOUT>(a, st);
    case 11: return launch_order<11, IO, ZIN, ZOUT>(a, st);
    case 12: return launch_order<12, IO, ZIN, ZOUT>(a, st);
    case 13: return launch_order<13, IO, ZIN, ZOUT>(a, st);
    case 14: return launch_order<14, IO, ZIN, ZOUT>(a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

// float32 activations (z in float32 throughout)
hyena_status_t dispatch_order_f32(int log2m, const Fused1dOrderArgs& a, cudaStream_t st);
// bf16 activations: first order (v bf16 -> z float32), middle orders
// (float32 -> float32), last order (float32 -> y bf16)
hyena_status_t dispatch_order_bf16_first(int log2m, const Fused1dOrderArgs& a, cudaStream_t st);
hyena_status_t dispatch_order_bf16_mid(int log2m, const Fused1dOrderArgs& a, cudaStream_t st);
hyena_status_t dispatch_order_bf16_last(int log2m, const Fused1dOrderArgs& a, cudaStream_t st);

}  // namespace hyena
