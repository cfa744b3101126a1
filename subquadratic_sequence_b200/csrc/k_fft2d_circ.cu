// Circular 2-D: the column launches of H-point transforms, the forward for
// both activation types and the circular 2-D filter spectra.
#include "k_fft2d.cuh"

namespace hyena {

// mode 0: full column step; 1: forward columns; 2: inverse columns
template <int LOG2H>
hyena_status_t launch_cols2d_circ_n(int mode, const Fft2dArgs& a, cudaStream_t st)
{
    using CL = Fft2dCols<LOG2H, false>;
    const unsigned grid = (unsigned)((long)a.nq * (a.W / CL::TC));
    if (mode == 1) return launch(fft2d_col_kernel<LOG2H, 1, false>, grid, CL::THREADS, CL::SMEM, st, a, false);
    if (mode == 2) return launch(fft2d_col_kernel<LOG2H, 2, false>, grid, CL::THREADS, CL::SMEM, st, a, false);
    return launch(fft2d_col_kernel<LOG2H, 0, false>, grid, CL::THREADS, CL::SMEM, st, a, false);
}

hyena_status_t launch_cols2d_circ(int log2h, int mode, const Fft2dArgs& a, cudaStream_t st)
{
    switch (log2h) {             // H-point columns
    case 4: return launch_cols2d_circ_n<4>(mode, a, st);
    case 5: return launch_cols2d_circ_n<5>(mode, a, st);
    case 6: return launch_cols2d_circ_n<6>(mode, a, st);
    case 7: return launch_cols2d_circ_n<7>(mode, a, st);
    case 8: return launch_cols2d_circ_n<8>(mode, a, st);
    case 9: return launch_cols2d_circ_n<9>(mode, a, st);
    case 10: return launch_cols2d_circ_n<10>(mode, a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t dispatch_fft2d_circ_f32(int log2m, int log2h, const Fft2dArgs& a, int N, float2* scratch,
                                       cudaStream_t st)
{
    return dispatch_fft2d_circ<float>(log2m, log2h, a, N, scratch, st);
}

hyena_status_t dispatch_fft2d_circ_bf16(int log2m, int log2h, const Fft2dArgs& a, int N, float2* scratch,
                                        cudaStream_t st)
{
    return dispatch_fft2d_circ<__nv_bfloat16>(log2m, log2h, a, N, scratch, st);
}

// circular 2-D spectra: forward rows of every filter into the H rows of
// its spectrum, then forward H-point columns in place
template <int LOG2M>
hyena_status_t run_rfft2d_circ(const Fft2dArgs& a, int log2h, cudaStream_t st)
{
    hyena_status_t s = launch_rows2d<LOG2M, float, 3, false>(a, st);
    return s == HYENA_OK ? launch_cols2d_circ(log2h, 1, a, st) : s;
}

hyena_status_t dispatch_rfft2d_circ(int log2m, int log2h, const Fft2dArgs& a, cudaStream_t st)
{
    switch (log2m) {
    case 4: return run_rfft2d_circ<4>(a, log2h, st);
    case 5: return run_rfft2d_circ<5>(a, log2h, st);
    case 6: return run_rfft2d_circ<6>(a, log2h, st);
    case 7: return run_rfft2d_circ<7>(a, log2h, st);
    case 8: return run_rfft2d_circ<8>(a, log2h, st);
    case 9: return run_rfft2d_circ<9>(a, log2h, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
