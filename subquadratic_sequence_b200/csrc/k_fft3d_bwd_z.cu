// z launches of the 3-D backward.
#include "k_fft3d_bwd.cuh"

namespace hyena {

template <int LOG2Z2, bool PAD>
hyena_status_t launch_bwd_z3d_n(int mode, const Bwd2dArgs& a, cudaStream_t st)
{
    using ZL = Fft3dZ<LOG2Z2, PAD>;
    const Fft2dArgs& f = a.f;
    const long H2 = (PAD ? 2L : 1L) * f.Hp;
    const long reg = H2 * (f.W / ZL::TC);                // regular CTAs per channel or spectrum
    if (mode == 2)
        return launch(fft3d_bwd_z_kernel<LOG2Z2, 2, PAD>, (unsigned)(f.nq * reg), ZL::THREADS, ZL::SMEM, st, a,
                      false);
    // channels the wave touches (volumes are channel-major), each with its
    // regular CTAs and its slot-0 pair CTAs
    const long nch = (long)(f.q0 + f.nq - 1) / f.B - f.q0 / f.B + 1;
    const long npair = (H2 / 2 + 1 + ZL::TC / 2 - 1) / (ZL::TC / 2);
    if (mode == 0)
        return launch(fft3d_bwd_z_kernel<LOG2Z2, 0, PAD>, (unsigned)(nch * (reg + npair)), ZL::THREADS, ZL::SMEM,
                      st, a, false);
    return launch(fft3d_bwd_z_kernel<LOG2Z2, 1, PAD>, (unsigned)(nch * (reg + npair)), ZL::THREADS, ZL::SMEM, st,
                  a, false);
}

hyena_status_t launch_bwd_z3d(int log2z, int mode, const Bwd2dArgs& a, cudaStream_t st)
{
    switch (log2z + 1) {          // 2Z-point transforms
    case 5: return launch_bwd_z3d_n<5, true>(mode, a, st);
    case 6: return launch_bwd_z3d_n<6, true>(mode, a, st);
    case 7: return launch_bwd_z3d_n<7, true>(mode, a, st);
    case 8: return launch_bwd_z3d_n<8, true>(mode, a, st);
    case 9: return launch_bwd_z3d_n<9, true>(mode, a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t launch_bwd_z3d_circ(int log2z, int mode, const Bwd2dArgs& a, cudaStream_t st)
{
    switch (log2z) {              // Z-point transforms
    case 4: return launch_bwd_z3d_n<4, false>(mode, a, st);
    case 5: return launch_bwd_z3d_n<5, false>(mode, a, st);
    case 6: return launch_bwd_z3d_n<6, false>(mode, a, st);
    case 7: return launch_bwd_z3d_n<7, false>(mode, a, st);
    case 8: return launch_bwd_z3d_n<8, false>(mode, a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
