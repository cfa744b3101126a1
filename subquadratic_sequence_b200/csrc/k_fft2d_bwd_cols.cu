// Column launches of the 2-D backward.
#include "k_fft2d_bwd.cuh"

namespace hyena {

template <int LOG2H2, bool PAD = true>
hyena_status_t launch_bwd_cols2d_n(int mode, const Bwd2dArgs& a, cudaStream_t st)
{
    using CL = Fft2dCols<LOG2H2, PAD>;
    const Fft2dArgs& f = a.f;
    const long per_unit = f.W / CL::TC;
    if (mode == 0)
        return launch(fft2d_bwd_col_kernel<LOG2H2, 0, PAD>, (unsigned)(f.nq * per_unit), CL::THREADS, CL::SMEM, st,
                      a, false);
    if (mode == 1) {
        // channels the wave touches (images are channel-major)
        const long nch = (long)(f.q0 + f.nq - 1) / f.B - f.q0 / f.B + 1;
        return launch(fft2d_bwd_col_kernel<LOG2H2, 1, PAD>, (unsigned)(nch * per_unit), CL::THREADS, CL::SMEM, st,
                      a, false);
    }
    return launch(fft2d_bwd_col_kernel<LOG2H2, 2, PAD>, (unsigned)(f.nq * per_unit), CL::THREADS, CL::SMEM, st, a,
                  false);
}

// circular mode: H-point columns, H in [16, 1024]
hyena_status_t launch_bwd_cols2d_circ(int log2h, int mode, const Bwd2dArgs& a, cudaStream_t st)
{
    switch (log2h) {
    case 4: return launch_bwd_cols2d_n<4, false>(mode, a, st);
    case 5: return launch_bwd_cols2d_n<5, false>(mode, a, st);
    case 6: return launch_bwd_cols2d_n<6, false>(mode, a, st);
    case 7: return launch_bwd_cols2d_n<7, false>(mode, a, st);
    case 8: return launch_bwd_cols2d_n<8, false>(mode, a, st);
    case 9: return launch_bwd_cols2d_n<9, false>(mode, a, st);
    case 10: return launch_bwd_cols2d_n<10, false>(mode, a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t launch_bwd_cols2d(int log2h, int mode, const Bwd2dArgs& a, cudaStream_t st)
{
    switch (log2h + 1) {          // 2H-point columns
    case 5: return launch_bwd_cols2d_n<5>(mode, a, st);
    case 6: return launch_bwd_cols2d_n<6>(mode, a, st);
    case 7: return launch_bwd_cols2d_n<7>(mode, a, st);
    case 8: return launch_bwd_cols2d_n<8>(mode, a, st);
    case 9: return launch_bwd_cols2d_n<9>(mode, a, st);
    case 10: return launch_bwd_cols2d_n<10>(mode, a, st);
    case 11: return launch_bwd_cols2d_n<11>(mode, a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
