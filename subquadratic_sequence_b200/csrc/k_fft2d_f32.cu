// 2-D forward with float32 activations; 2-D filter spectra; the column
// launches shared by both.
#include "k_fft2d.cuh"

namespace hyena {

// mode 0: full column step; 1: forward columns of planes; 2: inverse
// columns of planes (nq images or planes, one column block per CTA)
template <int LOG2H2>
hyena_status_t launch_cols2d_n(int mode, const Fft2dArgs& a, cudaStream_t st)
{
    using CL = Fft2dCols<LOG2H2>;
    const unsigned grid = (unsigned)((long)a.nq * (a.W / CL::TC));
    if (mode == 1) return launch(fft2d_col_kernel<LOG2H2, 1>, grid, CL::THREADS, CL::SMEM, st, a, false);
    if (mode == 2) return launch(fft2d_col_kernel<LOG2H2, 2>, grid, CL::THREADS, CL::SMEM, st, a, false);
    return launch(fft2d_col_kernel<LOG2H2, 0>, grid, CL::THREADS, CL::SMEM, st, a, false);
}

hyena_status_t launch_cols2d(int log2h, int mode, const Fft2dArgs& a, cudaStream_t st)
{
    switch (log2h + 1) {          // 2H-point columns
    case 5: return launch_cols2d_n<5>(mode, a, st);
    case 6: return launch_cols2d_n<6>(mode, a, st);
    case 7: return launch_cols2d_n<7>(mode, a, st);
    case 8: return launch_cols2d_n<8>(mode, a, st);
    case 9: return launch_cols2d_n<9>(mode, a, st);
    case 10: return launch_cols2d_n<10>(mode, a, st);
    case 11: return launch_cols2d_n<11>(mode, a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t dispatch_fft2d_f32(int log2w, int log2h, const Fft2dArgs& a, int N, float2* scratch,
                                  cudaStream_t st)
{
    return dispatch_fft2d<float>(log2w, log2h, a, N, scratch, st);
}

// 2-D spectra: forward rows of every filter into rows y < H of the packed
// spectra, then forward columns in place (all 2H rows written)
template <int LOG2W>
hyena_status_t run_rfft2d(Fft2dArgs a, int log2h, cudaStream_t st)
{
    hyena_status_t s = launch_rows2d<LOG2W, float, 3>(a, st);
    return s == HYENA_OK ? launch_cols2d(log2h, 1, a, st) : s;
}

hyena_status_t dispatch_rfft2d(int log2w, int log2h, const Fft2dArgs& a, cudaStream_t st)
{
    switch (log2w) {
    case 4: return run_rfft2d<4>(a, log2h, st);
    case 5: return run_rfft2d<5>(a, log2h, st);
    case 6: return run_rfft2d<6>(a, log2h, st);
    case 7: return run_rfft2d<7>(a, log2h, st);
    case 8: return run_rfft2d<8>(a, log2h, st);
    case 9: return run_rfft2d<9>(a, log2h, st);
    case 10: return run_rfft2d<10>(a, log2h, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
