// k_fft3d_bwd.cuh -- launch sequence of the 3-D backward, included by one
// .cu file per activation type.
#pragma once

#include "fft3d_bwd.cuh"
#include "k_fft2d_bwd.cuh"
#include "k_fft3d.cuh"

namespace hyena {

// z launches of the backward (log2z = log2 Z): mode 0 (A) and 1 (B) per
// channel of the wave, 2 per accumulated spectrum (f.nq of them)
hyena_status_t launch_bwd_z3d(int log2z, int mode, const Bwd2dArgs& a, cudaStream_t st);
hyena_status_t launch_bwd_z3d_circ(int log2z, int mode, const Bwd2dArgs& a, cudaStream_t st);

// The whole 3-D backward, wave by wave (A: the forward again, saving the
// spectra Z_n and the c_n; B: the orders in reverse), then dh and db from
// the accumulated spectra.  The row kernels see Z * H rows a volume; the
// column kernels see the wave's planes as images.
template <int LOG2W, typename IO, bool PAD = true>
hyena_status_t run_bwd3d(Bwd2dArgs a, int N, int log2h, int log2z, cudaStream_t st)
{
    using F1 = Fft1d<LOG2W, PAD>;
    Fft2dArgs& f = a.f;
    const int Z = f.zp, H = f.Hp;
    const long nimg = (long)f.B * f.C;
    const long per = a.wcap;
    const long sets = f.Hs_bstride != 0 ? f.B : 1;
    const size_t vol = (size_t)(PAD ? 4 : 1) * Z * H * f.W;   // spectrum slots per volume
    auto zstep = [&](int mode) {
        return PAD ? launch_bwd_z3d(log2z, mode, a, st) : launch_bwd_z3d_circ(log2z, mode, a, st);
    };
    auto planes = [&](int mode) {                               // forward (1) / inverse (2) columns
        Fft2dArgs pl = f;
        pl.q0 = 0;
        pl.nq = f.nq * Z;
        pl.zp = 0;
        pl.H = H;
        return launch_cols<PAD>(log2h, mode, pl, st);
    };
    a.N = N;
    f.H = Z * H;
    const cudaError_t e = cudaMemsetAsync(a.acc, 0, sizeof(float2) * (size_t)sets * N * f.C * vol, st);
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
            s = planes(1);
            if (s == HYENA_OK) s = zstep(0);
            if (s == HYENA_OK) s = planes(2);
            if (s == HYENA_OK) s = launch_bwd_rows2d<LOG2W, IO, 0, PAD>(a, st);
        }
        // B: the orders in reverse
        for (int n = N - 1; n >= 0 && s == HYENA_OK; --n) {
            f.n = n;
            a.first = n == N - 1;
            s = launch_bwd_rows2d<LOG2W, IO, 1, PAD>(a, st);
            if (s == HYENA_OK) s = planes(1);
            if (s == HYENA_OK) s = zstep(1);
            if (s == HYENA_OK) s = planes(2);
        }
        if (s == HYENA_OK) s = launch_bwd_rows2d<LOG2W, IO, 2, PAD>(a, st);
        if (s != HYENA_OK) return s;
    }
    // dh_n, db_n: inverse z transforms (planes z < Z), inverse columns of
    // those planes (padded: plane q is plane q % Z of spectrum q / Z at a
    // pitch of 2Z planes), inverse rows
    f.q0 = 0;
    f.nq = (int)(sets * N * f.C);
    hyena_status_t s = zstep(2);
    if (s == HYENA_OK) {
        Fft2dArgs pl = f;
        pl.S = a.acc;
        pl.q0 = 0;
        pl.nq = f.nq * Z;
        pl.zp = PAD ? Z : 0;
        pl.H = H;
        s = launch_cols<PAD>(log2h, 2, pl, st);
    }
    if (s == HYENA_OK) s = launch_bwd_rows2d<LOG2W, IO, 3, PAD>(a, st);
    if (s == HYENA_OK && f.Hs_bstride != 0)   // per-sample: db from the B lag-0 values
        s = launch(db2d_sum_kernel<PAD>, (unsigned)((N * f.C + 255) / 256), 256, 0, st, a);
    return s;
}

// log2m: log2 of the slots per row (W padded, W/2 circular)
template <typename IO>
hyena_status_t dispatch_bwd3d(int log2m, int log2h, int log2z, const Bwd2dArgs& a, int N, cudaStream_t st,
                              bool pad)
{
    if (!pad) {
        switch (log2m) {
        case 4: return run_bwd3d<4, IO, false>(a, N, log2h, log2z, st);
        case 5: return run_bwd3d<5, IO, false>(a, N, log2h, log2z, st);
        case 6: return run_bwd3d<6, IO, false>(a, N, log2h, log2z, st);
        case 7: return run_bwd3d<7, IO, false>(a, N, log2h, log2z, st);
        default: return HYENA_ERR_UNSUPPORTED;
        }
    }
    switch (log2m) {
    case 4: return run_bwd3d<4, IO>(a, N, log2h, log2z, st);
    case 5: return run_bwd3d<5, IO>(a, N, log2h, log2z, st);
    case 6: return run_bwd3d<6, IO>(a, N, log2h, log2z, st);
    case 7: return run_bwd3d<7, IO>(a, N, log2h, log2z, st);
    case 8: return run_bwd3d<8, IO>(a, N, log2h, log2z, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t dispatch_bwd3d_f32(int log2m, int log2h, int log2z, const Bwd2dArgs& a, int N, cudaStream_t st,
                                  bool pad);
hyena_status_t dispatch_bwd3d_bf16(int log2m, int log2h, int log2z, const Bwd2dArgs& a, int N, cudaStream_t st,
                                   bool pad);

}  // namespace hyena
