// k_circular.cuh -- launchers of the circular (unpadded) 1-D mode, included
// by one .cu file per activation type and by the spectrum file.  A real
// sequence of length L is the packed complex sequence of M = L/2 points:
// the same single-CTA kernels with PAD = false.
#pragma once

#include "launch.cuh"

namespace hyena {

constexpr int kMinLog2Circ = 4, kMaxLog2Circ = 13;   // M = L/2 in [16, 8192]: 32 <= L <= 16384

// PS: a spectrum set per sample (input-dependent filters)
template <int LOG2M, typename IO, bool PS = false>
hyena_status_t launch_fused_circ(const Fused1dArgs& a, cudaStream_t st)
{
    using F = Fft1d<LOG2M, false>;
    const long BD = (long)a.B * a.D;
    return launch(fused1d_kernel<LOG2M, IO, false, PS>, (unsigned)((BD + F::G - 1) / F::G), F::THREADS,
                  F::SMEM_BYTES, st, a);
}

template <typename IO, bool PS = false>
hyena_status_t dispatch_fused_circ(int log2m, const Fused1dArgs& a, cudaStream_t st)
{
    switch (log2m) {
    case 4: return launch_fused_circ<4, IO, PS>(a, st);
    case 5: return launch_fused_circ<5, IO, PS>(a, st);
    case 6: return launch_fused_circ<6, IO, PS>(a, st);
    case 7: return launch_fused_circ<7, IO, PS>(a, st);
    case 8: return launch_fused_circ<8, IO, PS>(a, st);
    case 9: return launch_fused_circ<9, IO, PS>(a, st);
    case 10: return launch_fused_circ<10, IO, PS>(a, st);
    case 11: return launch_fused_circ<11, IO, PS>(a, st);
    case 12: return launch_fused_circ<12, IO, PS>(a, st);
    case 13: return launch_fused_circ<13, IO, PS>(a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t dispatch_fused_circ_f32(int log2m, const Fused1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_fused_circ_bf16(int log2m, const Fused1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_fused_circ_ps_f32(int log2m, const Fused1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_fused_circ_ps_bf16(int log2m, const Fused1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_rfft_circ(int log2m, const Rfft1dArgs& a, cudaStream_t st);

}  // namespace hyena
