// k_fft2d.cuh -- launch sequences of the 2-D path, included by one .cu
// file per activation type.
#pragma once

#include "fft2d.cuh"
#include "launch.cuh"

namespace hyena {

constexpr int kMinLog2W2d = 4, kMaxLog2W2d = 10;    // W in [16, 1024]
constexpr int kMinLog2H2d = 4, kMaxLog2H2d = 10;    // H in [16, 1024] (2H-point columns)

// images per wave of the 2-D path (scratch = wave * H * W complex)
inline long wave_images(long nimg, long H, long W)
{
    long per = (long)(kWaveScratchBytes / (sizeof(float2) * (size_t)H * W));
    if (per < 1) per = 1;
    return nimg < per ? nimg : per;
}

// column launches: one column FFT per slot column, of 2H points (the log2
// given is log2 H) or, circular, of H points
hyena_status_t launch_cols2d(int log2h, int mode, const Fft2dArgs& a, cudaStream_t st);
hyena_status_t launch_cols2d_circ(int log2h, int mode, const Fft2dArgs& a, cudaStream_t st);

template <int LOG2M, typename IO, int MODE, bool PAD = true>
hyena_status_t launch_rows2d(const Fft2dArgs& a, cudaStream_t st)
{
    using F = Fft1d<LOG2M, PAD>;
    const long rows = (long)a.nq * a.H;
    return launch(fft2d_row_kernel<LOG2M, IO, MODE, PAD>, (unsigned)((rows + F::G - 1) / F::G), F::THREADS,
                  F::SMEM_BYTES_FFT, st, a, false);
}

// the order-N 2-D forward over B*C images, wave by wave
template <int LOG2W, typename IO>
hyena_status_t run_fft2d(Fft2dArgs a, int N, int log2h, float2* scratch, cudaStream_t st)
{
    const long nimg = (long)a.B * a.C, per = wave_images(nimg, a.H, a.W);
    a.S = scratch;
    for (long q0 = 0; q0 < nimg; q0 += per) {
        a.q0 = (int)q0;
        a.nq = (int)(nimg - q0 < per ? nimg - q0 : per);
        a.n = 0;
        hyena_status_t s = launch_rows2d<LOG2W, IO, 0>(a, st);
        for (int n = 0; n < N && s == HYENA_OK; ++n) {
            a.n = n;
            s = launch_cols2d(log2h, 0, a, st);
            if (s != HYENA_OK) break;
            s = n + 1 < N ? launch_rows2d<LOG2W, IO, 1>(a, st) : launch_rows2d<LOG2W, IO, 2>(a, st);
        }
        if (s != HYENA_OK) return s;
    }
    return HYENA_OK;
}

// the order-N circular 2-D forward (rows of W = 2M values, M slots; H-point
// columns): the same sequence without padding
template <int LOG2M, typename IO>
hyena_status_t run_fft2d_circ(Fft2dArgs a, int N, int log2h, float2* scratch, cudaStream_t st)
{
    const long nimg = (long)a.B * a.C, per = wave_images(nimg, a.H, a.W);
    a.S = scratch;
    for (long q0 = 0; q0 < nimg; q0 += per) {
        a.q0 = (int)q0;
        a.nq = (int)(nimg - q0 < per ? nimg - q0 : per);
        a.n = 0;
        hyena_status_t s = launch_rows2d<LOG2M, IO, 0, false>(a, st);
        for (int n = 0; n < N && s == HYENA_OK; ++n) {
            a.n = n;
            s = launch_cols2d_circ(log2h, 0, a, st);
            if (s != HYENA_OK) break;
            s = n + 1 < N ? launch_rows2d<LOG2M, IO, 1, false>(a, st) : launch_rows2d<LOG2M, IO, 2, false>(a, st);
        }
        if (s != HYENA_OK) return s;
    }
    return HYENA_OK;
}

template <typename IO>
hyena_status_t dispatch_fft2d_circ(int log2m, int log2h, const Fft2dArgs& a, int N, float2* scratch,
                                   cudaStream_t st)
{
    switch (log2m) {
    case 4: return run_fft2d_circ<4, IO>(a, N, log2h, scratch, st);
    case 5: return run_fft2d_circ<5, IO>(a, N, log2h, scratch, st);
    case 6: return run_fft2d_circ<6, IO>(a, N, log2h, scratch, st);
    case 7: return run_fft2d_circ<7, IO>(a, N, log2h, scratch, st);
    case 8: return run_fft2d_circ<8, IO>(a, N, log2h, scratch, st);
    case 9: return run_fft2d_circ<9, IO>(a, N, log2h, scratch, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

template <typename IO>
hyena_status_t dispatch_fft2d(int log2w, int log2h, const Fft2dArgs& a, int N, float2* scratch,
                              cudaStream_t st)
{
    switch (log2w) {
    case 4: return run_fft2d<4, IO>(a, N, log2h, scratch, st);
    case 5: return run_fft2d<5, IO>(a, N, log2h, scratch, st);
    case 6: return run_fft2d<6, IO>(a, N, log2h, scratch, st);
    case 7: return run_fft2d<7, IO>(a, N, log2h, scratch, st);
    case 8: return run_fft2d<8, IO>(a, N, log2h, scratch, st);
    case 9: return run_fft2d<9, IO>(a, N, log2h, scratch, st);
    case 10: return run_fft2d<10, IO>(a, N, log2h, scratch, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t dispatch_fft2d_f32(int log2w, int log2h, const Fft2dArgs& a, int N, float2* scratch,
                                  cudaStream_t st);
hyena_status_t dispatch_fft2d_bf16(int log2w, int log2h, const Fft2dArgs& a, int N, float2* scratch,
                                   cudaStream_t st);
hyena_status_t dispatch_rfft2d(int log2w, int log2h, const Fft2dArgs& a, cudaStream_t st);
hyena_status_t dispatch_fft2d_circ_f32(int log2m, int log2h, const Fft2dArgs& a, int N, float2* scratch,
                                       cudaStream_t st);
hyena_status_t dispatch_fft2d_circ_bf16(int log2m, int log2h, const Fft2dArgs& a, int N, float2* scratch,
                                        cudaStream_t st);
hyena_status_t dispatch_rfft2d_circ(int log2m, int log2h, const Fft2dArgs& a, cudaStream_t st);

}  // namespace hyena
