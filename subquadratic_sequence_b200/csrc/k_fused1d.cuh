// k_fused1d.cuh -- launchers of the single-CTA fused forward, included by
// one .cu file per activation type.
#pragma once

#include "launch.cuh"

namespace hyena {

template <int LOG2M, typename IO, bool PS>
hyena_status_t launch_fused(const Fused1dArgs& a, cudaStream_t st)
{
    using F = Fft1d<LOG2M>;
    const long BD = (long)a.B * a.D;
    return launch(fused1d_kernel<LOG2M, IO, true, PS>, (unsigned)((BD + F::G - 1) / F::G), F::THREADS,
                  F::SMEM_BYTES, st, a);
}

// PS: per-sample spectra (a.H_bstride != 0)
template <typename IO, bool PS>
hyena_status_t dispatch_fused(int log2m, const Fused1dArgs& a, cudaStream_t st)
{
    switch (log2m) {
    case 4: return launch_fused<4, IO, PS>(a, st);
    case 5: return launch_fused<5, IO, PS>(a, st);
    case 6: return launch_fused<6, IO, PS>(a, st);
    case 7: return launch_fused<7, IO, PS>(a, st);
    case 8: return launch_fused<8, IO, PS>(a, st);
    case 9: return launch_fused<9, IO, PS>(a, st);
    case 10: return launch_fused<10, IO, PS>(a, st);
    case 11: return launch_fused<11, IO, PS>(a, st);
    case 12: return launch_fused<12, IO, PS>(a, st);
    case 13: return launch_fused<13, IO, PS>(a, st);
    case 14: return launch_fused<14, IO, PS>(a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
