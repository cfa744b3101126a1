// k_fft3d.cuh -- launch sequences of the 3-D path, included by one .cu file
// per activation type and by the spectrum file.
#pragma once

#include "fft3d.cuh"
#include "k_fft2d.cuh"

namespace hyena {

constexpr int kMinLog2_3d = 4, kMaxLog2_3d = 8;      // Z, H, W in [16, 256]

hyena_status_t launch_z3d(int log2z, int mode, const Fft2dArgs& a, cudaStream_t st);

// images per wave of the 3-D path (scratch = Z planes of 2H x W slots each)
inline long wave_images_3d(long nimg, long Z, long H, long W)
{
    long per = (long)(kWaveScratchBytes / (sizeof(float2) * (size_t)Z * 2 * H * W));
    if (per < 1) per = 1;
    return nimg < per ? nimg : per;
}

// the order-N 3-D forward over B*C images, wave by wave
template <int LOG2W, typename IO>
hyena_status_t run_fft3d(Fft2dArgs a, int N, int log2h, int log2z, float2* scratch, cudaStream_t st)
{
    const int Z = a.zp, H = a.Hp;
    const long nimg = (long)a.B * a.C, per = wave_images_3d(nimg, Z, H, a.W);
    a.S = scratch;
    a.H = Z * H;                                     // rows per image for the row kernel
    for (long q0 = 0; q0 < nimg; q0 += per) {
        a.q0 = (int)q0;
        a.nq = (int)(nimg - q0 < per ? nimg - q0 : per);
        a.n = 0;
        Fft2dArgs pl = a;                            // the wave's planes, contiguous, for the columns
        pl.q0 = 0;
        pl.nq = a.nq * Z;
        pl.zp = 0;
        pl.H = H;
        hyena_status_t s = launch_rows2d<LOG2W, IO, 0>(a, st);
        if (s == HYENA_OK) s = launch_cols2d(log2h, 1, pl, st);
        for (int n = 0; n < N && s == HYENA_OK; ++n) {
            a.n = n;
            s = launch_z3d(log2z, 0, a, st);
            if (s == HYENA_OK) s = launch_cols2d(log2h, 2, pl, st);
            if (s != HYENA_OK) break;
            if (n + 1 < N) {
                s = launch_rows2d<LOG2W, IO, 1>(a, st);
                if (s == HYENA_OK) s = launch_cols2d(log2h, 1, pl, st);
            } else {
                s = launch_rows2d<LOG2W, IO, 2>(a, st);
            }
        }
        if (s != HYENA_OK) return s;
    }
    return HYENA_OK;
}

template <typename IO>
hyena_status_t dispatch_fft3d(int log2w, int log2h, int log2z, const Fft2dArgs& a, int N, float2* scratch,
                              cudaStream_t st)
{
    switch (log2w) {
    case 4: return run_fft3d<4, IO>(a, N, log2h, log2z, scratch, st);
    case 5: return run_fft3d<5, IO>(a, N, log2h, log2z, scratch, st);
    case 6: return run_fft3d<6, IO>(a, N, log2h, log2z, scratch, st);
    case 7: return run_fft3d<7, IO>(a, N, log2h, log2z, scratch, st);
    case 8: return run_fft3d<8, IO>(a, N, log2h, log2z, scratch, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t dispatch_fft3d_f32(int log2w, int log2h, int log2z, const Fft2dArgs& a, int N,
                                  float2* scratch, cudaStream_t st);
hyena_status_t dispatch_fft3d_bf16(int log2w, int log2h, int log2z, const Fft2dArgs& a, int N,
                                   float2* scratch, cudaStream_t st);
hyena_status_t dispatch_rfft3d(int log2w, int log2h, int log2z, const Fft2dArgs& a, cudaStream_t st);

}  // namespace hyena
