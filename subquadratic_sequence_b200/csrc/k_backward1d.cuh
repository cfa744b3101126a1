// k_backward1d.cuh -- launchers of the 1-D backward pass, included by one
// .cu file per activation type.
#pragma once

#include "backward1d.cuh"
#include "launch.cuh"

namespace hyena {

template <int LOG2M, typename IO, bool PS, bool PAD>
hyena_status_t launch_backward(const Backward1dArgs& a, cudaStream_t st)
{
    using F = Fft1d<LOG2M, PAD>;
    hyena_status_t s = launch(backward1d_kernel<LOG2M, IO, PS, PAD>, (unsigned)((a.D + F::G - 1) / F::G),
                              F::THREADS, F::SMEM_BYTES, st, a);
    if (s != HYENA_OK) return s;
    const int rows = a.N * a.D;
    return launch(dh_finalize_kernel<LOG2M, PS, PAD>, (unsigned)((rows + F::G - 1) / F::G), F::THREADS,
                  F::SMEM_BYTES_FFT, st, a);
}

// PS: a spectrum set per sample (per-sample dh); PAD false: circular mode
// (log2m = log2(L/2) up to 13)
template <typename IO, bool PS = false, bool PAD = true>
hyena_status_t dispatch_backward(int log2m, const Backward1dArgs& a, cudaStream_t st)
{
    switch (log2m) {
    case 4: return launch_backward<4, IO, PS, PAD>(a, st);
    case 5: return launch_backward<5, IO, PS, PAD>(a, st);
    case 6: return launch_backward<6, IO, PS, PAD>(a, st);
    case 7: return launch_backward<7, IO, PS, PAD>(a, st);
    case 8: return launch_backward<8, IO, PS, PAD>(a, st);
    case 9: return launch_backward<9, IO, PS, PAD>(a, st);
    case 10: return launch_backward<10, IO, PS, PAD>(a, st);
    case 11: return launch_backward<11, IO, PS, PAD>(a, st);
    case 12: return launch_backward<12, IO, PS, PAD>(a, st);
    case 13: return launch_backward<13, IO, PS, PAD>(a, st);
    case 14:
        if constexpr (PAD) return launch_backward<14, IO, PS, PAD>(a, st);
        return HYENA_ERR_UNSUPPORTED;
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
