// k_fused1d.cuh -- launchers of the single-CTA fused forward, included by
// one .cu file per activation type.
#pragma once

#include "launch.cuh"

namespace hyena {

template <int LOG2M, typename IO>
hyena_status_t launch_fused(const Fused1dArgs& a, cudaStream_t st)
{
    using F = Fft1d<LOG2M>;
    const long BD = (long)a.B * a.D;
    return launch(fused1d_kernel<LOG2M, IO>, (unsigned)((BD + F::G - 1) / F::G), F::THREADS,
                  F::SMEM_BYTES, st, a);
}

template <typename IO>
hyena_status_t dispatch_fused(int log2m, const Fused1dArgs& a, cudaStream_t st)
{
    switch (log2m) {
    case 4: return launch_fused<4, IO>(a, st);
    case 5: return launch_fused<5, IO>(a, st);
    case 6: return launch_fused<6, IO>(a, st);
    case 7: return launch_fused<7, IO>(a, st);
    case 8: return launch_fused<8, IO>(a, st);
    case 9: return launch_fused<9, IO>(a, st);
    case 10: return launch_fused<10, IO>(a, st);
    case 11: return launch_fused<11, IO>(a, st);
    case 12: return launch_fused<12, IO>(a, st);
    case 13: return launch_fused<13, IO>(a, st);
    case 14: return launch_fused<14, IO>(a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
