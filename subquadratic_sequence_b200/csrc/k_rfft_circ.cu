// Spectra of unpadded filters (circular mode).
#include "k_circular.cuh"

namespace hyena {

template <int LOG2M>
hyena_status_t launch_rfft_circ(const Rfft1dArgs& a, cudaStream_t st)
{
    using F = Fft1d<LOG2M, false>;
    return launch(rfft1d_kernel<LOG2M, false>, (unsigned)((a.rows + F::G - 1) / F::G), F::THREADS,
                  F::SMEM_BYTES_FFT, st, a);
}

hyena_status_t dispatch_rfft_circ(int log2m, const Rfft1dArgs& a, cudaStream_t st)
{
    switch (log2m) {
    case 4: return launch_rfft_circ<4>(a, st);
    case 5: return launch_rfft_circ<5>(a, st);
    case 6: return launch_rfft_circ<6>(a, st);
    case 7: return launch_rfft_circ<7>(a, st);
    case 8: return launch_rfft_circ<8>(a, st);
    case 9: return launch_rfft_circ<9>(a, st);
    case 10: return launch_rfft_circ<10>(a, st);
    case 11: return launch_rfft_circ<11>(a, st);
    case 12: return launch_rfft_circ<12>(a, st);
    case 13: return launch_rfft_circ<13>(a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
