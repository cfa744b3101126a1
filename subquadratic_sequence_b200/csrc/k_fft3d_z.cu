// The z kernels of the 3-D path and the 3-D filter spectra.
#include "k_fft3d.cuh"

namespace hyena {

template <int LOG2Z2>
hyena_status_t launch_z3d_n(int mode, const Fft2dArgs& a, cudaStream_t st)
{
    using ZL = Fft3dZ<LOG2Z2>;
    const long reg = 2L * a.Hp * (a.W / ZL::TC);          // regular CTAs per image or channel
    if (mode == 1)
        return launch(fft3d_z_kernel<LOG2Z2, 1>, (unsigned)(a.nq * reg), ZL::THREADS, ZL::SMEM, st, a, false);
    // channels the wave touches (images are channel-major), each with its
    // regular CTAs and its pair CTAs
    const long nch = (long)(a.q0 + a.nq - 1) / a.B - a.q0 / a.B + 1;
    const long npair = (a.Hp + 1 + ZL::TC / 2 - 1) / (ZL::TC / 2);
    return launch(fft3d_z_kernel<LOG2Z2, 0>, (unsigned)(nch * (reg + npair)), ZL::THREADS, ZL::SMEM, st, a,
                  false);
}

hyena_status_t launch_z3d(int log2z, int mode, const Fft2dArgs& a, cudaStream_t st)
{
    switch (log2z + 1) {          // 2Z-point transforms
    case 5: return launch_z3d_n<5>(mode, a, st);
    case 6: return launch_z3d_n<6>(mode, a, st);
    case 7: return launch_z3d_n<7>(mode, a, st);
    case 8: return launch_z3d_n<8>(mode, a, st);
    case 9: return launch_z3d_n<9>(mode, a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

// 3-D spectra: forward rows of every filter plane into planes z < Z of the
// packed spectra [N*C][2Z][2H][W], forward columns of those planes, then
// the forward z transform of every slot (all 2Z planes written)
template <int LOG2W>
hyena_status_t rfft3d_w(int log2h, int log2z, Fft2dArgs a, cudaStream_t st)
{
    const int Z = a.zp, H = a.Hp;
    a.H = Z * H;
    hyena_status_t s = launch_rows2d<LOG2W, float, 3>(a, st);
    if (s != HYENA_OK) return s;
    Fft2dArgs pl = a;
    pl.nq = a.nq * Z;                    // planes, remapped to f * 2Z + z by the column kernel
    pl.H = H;
    s = launch_cols2d(log2h, 1, pl, st);
    if (s != HYENA_OK) return s;
    return launch_z3d(log2z, 1, a, st);
}

hyena_status_t dispatch_rfft3d(int log2w, int log2h, int log2z, const Fft2dArgs& a, cudaStream_t st)
{
    switch (log2w) {
    case 4: return rfft3d_w<4>(log2h, log2z, a, st);
    case 5: return rfft3d_w<5>(log2h, log2z, a, st);
    case 6: return rfft3d_w<6>(log2h, log2z, a, st);
    case 7: return rfft3d_w<7>(log2h, log2z, a, st);
    case 8: return rfft3d_w<8>(log2h, log2z, a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
