// k_fft2d_bwd.cuh -- launch sequence of the 2-D backward, included by one
// .cu file per activation type.
#pragma once

#include "fft2d_bwd.cuh"
#include "k_fft2d.cuh"

namespace hyena {

// column launches of the backward (log2h = log2 H; 2H-point columns, or
// H-point circular columns): mode 0 per image, 1 per channel of the wave,
// 2 per filter row
hyena_status_t launch_bwd_cols2d(int log2h, int mode, const Bwd2dArgs& a, cudaStream_t st);
hyena_status_t launch_bwd_cols2d_circ(int log2h, int mode, const Bwd2dArgs& a, cudaStream_t st);

template <int LOG2W, typename IO, int MODE, bool PAD>
hyena_status_t launch_bwd_rows2d(const Bwd2dArgs& a, cudaStream_t st)
{
    using F = Fft1d<LOG2W, PAD>;
    const long rows = (long)a.f.nq * a.f.H;
    return launch(fft2d_bwd_row_kernel<LOG2W, IO, MODE, PAD>, (unsigned)((rows + F::G - 1) / F::G), F::THREADS,
                  F::SMEM_BYTES_FFT, st, a, false);
}

// The whole backward: per wave the forward again (A) and the orders in
// reverse (B); then dh and db from the accumulated spectra (zeroed first).
// PAD false: circular mode (rows of W = 2 slots reals, H-point columns).
template <int LOG2W, typename IO, bool PAD = true>
hyena_status_t run_bwd2d(Bwd2dArgs a, int N, int log2h, cudaStream_t st)
{
    using F1 = Fft1d<LOG2W, PAD>;
    auto cols = [&](int mode) {
        return PAD ? launch_bwd_cols2d(log2h, mode, a, st) : launch_bwd_cols2d_circ(log2h, mode, a, st);
    };
    Fft2dArgs& f = a.f;
    const long nimg = (long)f.B * f.C;
    const long per = a.wcap;
    const long sets = f.Hs_bstride != 0 ? f.B : 1;            // dh spectra per (n, c)
    a.N = N;
    const cudaError_t e =
        cudaMemsetAsync(a.acc, 0, sizeof(float2) * (size_t)sets * N * f.C * (PAD ? 2 : 1) * f.H * f.W, st);
    if (e != cudaSuccess) return from_cuda(e);
    for (long q0 = 0; q0 < nimg; q0 += per) {
        f.q0 = (int)q0;
        f.nq = (int)(nimg - q0 < per ? nimg - q0 : per);
        f.n = 0;
        // A: the forward, saving Z_n and c_n
        hyena_status_t s = launch(fft2d_row_kernel<LOG2W, IO, 0, PAD>,
                                  (unsigned)(((long)f.nq * f.H + F1::G - 1) / F1::G),
                                  F1::THREADS, F1::SMEM_BYTES_FFT, st, f, false);
        for (int n = 0; n < N && s == HYENA_OK; ++n) {
            f.n = n;
            a.last = n + 1 == N;
            s = cols(0);
            if (s == HYENA_OK) s = launch_bwd_rows2d<LOG2W, IO, 0, PAD>(a, st);
        }
        // B: the orders in reverse
        for (int n = N - 1; n >= 0 && s == HYENA_OK; --n) {
            f.n = n;
            a.first = n == N - 1;
            s = launch_bwd_rows2d<LOG2W, IO, 1, PAD>(a, st);
            if (s == HYENA_OK) s = cols(1);
        }
        if (s == HYENA_OK) s = launch_bwd_rows2d<LOG2W, IO, 2, PAD>(a, st);
        if (s != HYENA_OK) return s;
    }
    // dh_n, db_n: inverse columns, then inverse rows, of the sets*N*C spectra
    f.q0 = 0;
    f.nq = (int)(sets * N * f.C);
    hyena_status_t s = cols(2);
    if (s == HYENA_OK) s = launch_bwd_rows2d<LOG2W, IO, 3, PAD>(a, st);
    if (s == HYENA_OK && f.Hs_bstride != 0)   // per-sample: db from the B lag-0 values (any B)
        s = launch(db2d_sum_kernel<PAD>, (unsigned)((N * f.C + 255) / 256), 256, 0, st, a);
    return s;
}

// circular mode: log2m = log2 of the slots per row (W/2), 4 .. 9
template <typename IO>
hyena_status_t dispatch_bwd2d_circ(int log2m, int log2h, const Bwd2dArgs& a, int N, cudaStream_t st)
{
    switch (log2m) {
    case 4: return run_bwd2d<4, IO, false>(a, N, log2h, st);
    case 5: return run_bwd2d<5, IO, false>(a, N, log2h, st);
    case 6: return run_bwd2d<6, IO, false>(a, N, log2h, st);
    case 7: return run_bwd2d<7, IO, false>(a, N, log2h, st);
    case 8: return run_bwd2d<8, IO, false>(a, N, log2h, st);
    case 9: return run_bwd2d<9, IO, false>(a, N, log2h, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

template <typename IO>
hyena_status_t dispatch_bwd2d(int log2w, int log2h, const Bwd2dArgs& a, int N, cudaStream_t st)
{
    switch (log2w) {
    case 4: return run_bwd2d<4, IO>(a, N, log2h, st);
    case 5: return run_bwd2d<5, IO>(a, N, log2h, st);
    case 6: return run_bwd2d<6, IO>(a, N, log2h, st);
    case 7: return run_bwd2d<7, IO>(a, N, log2h, st);
    case 8: return run_bwd2d<8, IO>(a, N, log2h, st);
    case 9: return run_bwd2d<9, IO>(a, N, log2h, st);
    case 10: return run_bwd2d<10, IO>(a, N, log2h, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t dispatch_bwd2d_f32(int log2w, int log2h, const Bwd2dArgs& a, int N, cudaStream_t st);
hyena_status_t dispatch_bwd2d_bf16(int log2w, int log2h, const Bwd2dArgs& a, int N, cudaStream_t st);
hyena_status_t dispatch_bwd2d_circ_f32(int log2m, int log2h, const Bwd2dArgs& a, int N, cudaStream_t st);
hyena_status_t dispatch_bwd2d_circ_bf16(int log2m, int log2h, const Bwd2dArgs& a, int N, cudaStream_t st);

}  // namespace hyena
