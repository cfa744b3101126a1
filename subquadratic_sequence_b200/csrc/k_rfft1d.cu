// Filter spectra for L <= 16384 (single CTA per filter row).
#include "launch.cuh"

namespace hyena {

template <int LOG2M>
hyena_status_t launch_rfft(const Rfft1dArgs& a, cudaStream_t st)
{
    using F = Fft1d<LOG2M>;
    return launch(rfft1d_kernel<LOG2M>, (unsigned)((a.rows + F::G - 1) / F::G), F::THREADS,
                  F::SMEM_BYTES_FFT, st, a);
}

hyena_status_t dispatch_rfft(int log2m, const Rfft1dArgs& a, cudaStream_t st)
{
    switch (log2m) {
    case 4: return launch_rfft<4>(a, st);
    case 5: return launch_rfft<5>(a, st);
    case 6: return launch_rfft<6>(a, st);
    case 7: return launch_rfft<7>(a, st);
    case 8: return launch_rfft<8>(a, st);
    case 9: return launch_rfft<9>(a, st);
    case 10: return launch_rfft<10>(a, st);
    case 11: return launch_rfft<11>(a, st);
    case 12: return launch_rfft<12>(a, st);
    case 13: return launch_rfft<13>(a, st);
    case 14: return launch_rfft<14>(a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
