// The z kernels of the 3-D path and the 3-D filter spectra.
#include "k_fft3d.cuh"

namespace hyena {

template <int LOG2Z2, bool PAD>
hyena_status_t launch_z3d_n(int mode, const Fft2dArgs& a, cudaStream_t st)
{
    using ZL = Fft3dZ<LOG2Z2, PAD>;
    const long H2 = (PAD ? 2L : 1L) * a.Hp;
    const long reg = H2 * (a.W / ZL::TC);                // regular CTAs per volume or channel
    if (mode == 1)
        return launch(fft3d_z_kernel<LOG2Z2, 1, PAD>, (unsigned)(a.nq * reg), ZL::THREADS, ZL::SMEM, st, a, false);
    // channels the wave touches (volumes are channel-major), each with its
    // regular CTAs and its pair CTAs
    const long nch = (long)(a.q0 + a.nq - 1) / a.B - a.q0 / a.B + 1;
    const long npair = (H2 / 2 + 1 + ZL::TC / 2 - 1) / (ZL::TC / 2);
    if (a.Hs_bstride != 0)            // a spectrum set per sample
        return launch(fft3d_z_kernel<LOG2Z2, 2, PAD>, (unsigned)(nch * (reg + npair)), ZL::THREADS, ZL::SMEM,
                      st, a, false);
    return launch(fft3d_z_kernel<LOG2Z2, 0, PAD>, (unsigned)(nch * (reg + npair)), ZL::THREADS, ZL::SMEM, st,
                  a, false);
}

hyena_status_t launch_z3d(int log2z, int mode, const Fft2dArgs& a, cudaStream_t st)
{
    switch (log2z + 1) {          // 2Z-point transforms
    case 5: return launch_z3d_n<5, true>(mode, a, st);
    case 6: return launch_z3d_n<6, true>(mode, a, st);
    case 7: return launch_z3d_n<7, true>(mode, a, st);
    case 8: return launch_z3d_n<8, true>(mode, a, st);
    case 9: return launch_z3d_n<9, true>(mode, a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t launch_z3d_circ(int log2z, int mode, const Fft2dArgs& a, cudaStream_t st)
{
    switch (log2z) {              // Z-point transforms
    case 4: return launch_z3d_n<4, false>(mode, a, st);
    case 5: return launch_z3d_n<5, false>(mode, a, st);
    case 6: return launch_z3d_n<6, false>(mode, a, st);
    case 7: return launch_z3d_n<7, false>(mode, a, st);
    case 8: return launch_z3d_n<8, false>(mode, a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

// 3-D spectra: forward rows of every filter plane into planes z < Z of the
// packed spectra [N*C][2Z][2H][W] (circular: all Z planes of [Z][H][W/2]),
// forward columns of those planes, then the forward z transform of every
// slot (all planes written)
template <int LOG2M, bool PAD>
hyena_status_t rfft3d_w(int log2h, int log2z, Fft2dArgs a, cudaStream_t st)
{
    const int Z = a.zp, H = a.Hp;
    a.H = Z * H;
    hyena_status_t s = launch_rows2d<LOG2M, float, 3, PAD>(a, st);
    if (s != HYENA_OK) return s;
    Fft2dArgs pl = a;
    pl.nq = a.nq * Z;                    // planes (padded: remapped to f * 2Z + z by the column kernel)
    pl.H = H;
    s = launch_cols<PAD>(log2h, 1, pl, st);
    if (s != HYENA_OK) return s;
    return launch_z<PAD>(log2z, 1, a, st);
}

hyena_status_t dispatch_rfft3d(int log2m, int log2h, int log2z, const Fft2dArgs& a, cudaStream_t st, bool pad)
{
    if (!pad) {
        switch (log2m) {
        case 4: return rfft3d_w<4, false>(log2h, log2z, a, st);
        case 5: return rfft3d_w<5, false>(log2h, log2z, a, st);
        case 6: return rfft3d_w<6, false>(log2h, log2z, a, st);
        case 7: return rfft3d_w<7, false>(log2h, log2z, a, st);
        default: return HYENA_ERR_UNSUPPORTED;
        }
    }
    switch (log2m) {
    case 4: return rfft3d_w<4, true>(log2h, log2z, a, st);
    case 5: return rfft3d_w<5, true>(log2h, log2z, a, st);
    case 6: return rfft3d_w<6, true>(log2h, log2z, a, st);
    case 7: return rfft3d_w<7, true>(log2h, log2z, a, st);
    case 8: return rfft3d_w<8, true>(log2h, log2z, a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
