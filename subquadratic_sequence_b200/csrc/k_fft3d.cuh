// k_fft3d.cuh -- launch sequences of the 3-D path (padded and circular),
// included by one .cu file per activation type and by the spectrum file.
#pragma once

#include "fft3d.cuh"
#include "k_fft2d.cuh"

namespace hyena {

constexpr int kMinLog2_3d = 4, kMaxLog2_3d = 8;      // Z, H, W in [16, 256]

// z kernels: 2Z-point transforms (log2z = log2 Z) or, circular, Z-point
hyena_status_t launch_z3d(int log2z, int mode, const Fft2dArgs& a, cudaStream_t st);
hyena_status_t launch_z3d_circ(int log2z, int mode, const Fft2dArgs& a, cudaStream_t st);

template <bool PAD>
inline hyena_status_t launch_z(int log2z, int mode, const Fft2dArgs& a, cudaStream_t st)
{
    return PAD ? launch_z3d(log2z, mode, a, st) : launch_z3d_circ(log2z, mode, a, st);
}

template <bool PAD>
inline hyena_status_t launch_cols(int log2h, int mode, const Fft2dArgs& a, cudaStream_t st)
{
    return PAD ? launch_cols2d(log2h, mode, a, st) : launch_cols2d_circ(log2h, mode, a, st);
}

// volumes per wave of the 3-D path (scratch = Z planes of 2H x W slots
// each, or of H x W slots when circular; W here counts slots)
inline long wave_images_3d(long nimg, long Z, long H, long W, bool pad = true)
{
    long per = (long)(kWaveScratchBytes / (sizeof(float2) * (size_t)Z * (pad ? 2 : 1) * H * W));
    if (per < 1) per = 1;
    return nimg < per ? nimg : per;
}

// the order-N 3-D forward over B*C volumes, wave by wave (LOG2M: log2 of
// the slots per row)
template <int LOG2M, typename IO, bool PAD>
hyena_status_t run_fft3d(Fft2dArgs a, int N, int log2h, int log2z, float2* scratch, cudaStream_t st)
{
    const int Z = a.zp, H = a.Hp;
    const long nimg = (long)a.B * a.C, per = wave_images_3d(nimg, Z, H, a.W, PAD);
    a.S = scratch;
    a.H = Z * H;                                     // rows per volume for the row kernel
    for (long q0 = 0; q0 < nimg; q0 += per) {
        a.q0 = (int)q0;
        a.nq = (int)(nimg - q0 < per ? nimg - q0 : per);
        a.n = 0;
        Fft2dArgs pl = a;                            // the wave's planes, contiguous, for the columns
        pl.q0 = 0;
        pl.nq = a.nq * Z;
        pl.zp = 0;
        pl.H = H;
        hyena_status_t s = launch_rows2d<LOG2M, IO, 0, PAD>(a, st);
        if (s == HYENA_OK) s = launch_cols<PAD>(log2h, 1, pl, st);
        for (int n = 0; n < N && s == HYENA_OK; ++n) {
            a.n = n;
            s = launch_z<PAD>(log2z, 0, a, st);
            if (s == HYENA_OK) s = launch_cols<PAD>(log2h, 2, pl, st);
            if (s != HYENA_OK) break;
            if (n + 1 < N) {
                s = launch_rows2d<LOG2M, IO, 1, PAD>(a, st);
                if (s == HYENA_OK) s = launch_cols<PAD>(log2h, 1, pl, st);
            } else {
                s = launch_rows2d<LOG2M, IO, 2, PAD>(a, st);
            }
        }
        if (s != HYENA_OK) return s;
    }
    return HYENA_OK;
}

template <typename IO, bool PAD>
hyena_status_t dispatch_fft3d(int log2m, int log2h, int log2z, const Fft2dArgs& a, int N, float2* scratch,
                              cudaStream_t st)
{
    switch (log2m) {
    case 4: return run_fft3d<4, IO, PAD>(a, N, log2h, log2z, scratch, st);
    case 5: return run_fft3d<5, IO, PAD>(a, N, log2h, log2z, scratch, st);
    case 6: return run_fft3d<6, IO, PAD>(a, N, log2h, log2z, scratch, st);
    case 7: return run_fft3d<7, IO, PAD>(a, N, log2h, log2z, scratch, st);
    case 8:
        if constexpr (PAD) return run_fft3d<8, IO, PAD>(a, N, log2h, log2z, scratch, st);
        return HYENA_ERR_UNSUPPORTED;
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t dispatch_fft3d_f32(int log2w, int log2h, int log2z, const Fft2dArgs& a, int N,
                                  float2* scratch, cudaStream_t st, bool pad = true);
hyena_status_t dispatch_fft3d_bf16(int log2w, int log2h, int log2z, const Fft2dArgs& a, int N,
                                   float2* scratch, cudaStream_t st, bool pad = true);
hyena_status_t dispatch_rfft3d(int log2w, int log2h, int log2z, const Fft2dArgs& a, cudaStream_t st,
                               bool pad = true);

}  // namespace hyena
