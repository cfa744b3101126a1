// k_fourstep.cuh -- wave-by-wave launch sequences of the four-step path,
// included by one .cu file per activation type (and one for the spectra).
#pragma once

#include "launch.cuh"

namespace hyena {

// The order-N forward over B*D sequences, wave by wave: per wave one
// column launch (from v), then per order a row launch and a column launch.
// PAD false: circular mode (M-point transforms of 2M unpadded reals).
template <int LM1, int LM2, typename IO, bool PAD = true>
hyena_status_t run_fourstep(FourStepArgs a, int N, float2* scratch, cudaStream_t st)
{
    using FS = FourStep<LM1, LM2>;
    const long nseq = (long)a.B * a.D, per = wave_seqs(nseq, FS::M);
    a.S = scratch;
    a.n_last = N - 1;
    for (long q0 = 0; q0 < nseq; q0 += per) {
        const unsigned nq = (unsigned)(nseq - q0 < per ? nseq - q0 : per);
        a.q0 = (int)q0;
        a.n = 0;
        hyena_status_t s = launch(fourstep_col_kernel<LM1, LM2, IO, 0, PAD>, nq * FS::COL_CTAS_PER_SEQ,
                                  FS::COL_THREADS, FS::COL_SMEM, st, a);
        for (int n = 0; n < N && s == HYENA_OK; ++n) {
            a.n = n;
            s = launch(fourstep_row_kernel<LM1, LM2, false>, nq * FS::ROW_CTAS_PER_SEQ,
                       FS::ROW_THREADS, FS::ROW_SMEM, st, a);
            if (s != HYENA_OK) break;
            s = n + 1 < N ? launch(fourstep_col_kernel<LM1, LM2, IO, 1, PAD>, nq * FS::COL_CTAS_PER_SEQ,
                                   FS::COL_THREADS, FS::COL_SMEM, st, a)
                          : launch(fourstep_col_kernel<LM1, LM2, IO, 2, PAD>, nq * FS::COL_CTAS_PER_SEQ,
                                   FS::COL_THREADS, FS::COL_SMEM, st, a);
        }
        if (s != HYENA_OK) return s;
    }
    return HYENA_OK;
}

template <typename IO>
hyena_status_t dispatch_fourstep(int log2m, const FourStepArgs& a, int N, float2* scratch,
                                 cudaStream_t st)
{
    switch (log2m) {
    case 15: return run_fourstep<7, 8, IO>(a, N, scratch, st);
    case 16: return run_fourstep<8, 8, IO>(a, N, scratch, st);
    case 17: return run_fourstep<8, 9, IO>(a, N, scratch, st);
    case 18: return run_fourstep<8, 10, IO>(a, N, scratch, st);
    case 19: return run_fourstep<9, 10, IO>(a, N, scratch, st);
    case 20: return run_fourstep<10, 10, IO>(a, N, scratch, st);
    case 21: return run_fourstep<10, 11, IO>(a, N, scratch, st);
    case 22: return run_fourstep<11, 11, IO>(a, N, scratch, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

// circular mode: log2m = log2(L/2), 14 .. 21 (16384 < L <= 2^22)
template <typename IO>
hyena_status_t dispatch_fourstep_circ(int log2m, const FourStepArgs& a, int N, float2* scratch,
                                      cudaStream_t st)
{
    switch (log2m) {
    case 14: return run_fourstep<7, 7, IO, false>(a, N, scratch, st);
    case 15: return run_fourstep<7, 8, IO, false>(a, N, scratch, st);
    case 16: return run_fourstep<8, 8, IO, false>(a, N, scratch, st);
    case 17: return run_fourstep<8, 9, IO, false>(a, N, scratch, st);
    case 18: return run_fourstep<9, 9, IO, false>(a, N, scratch, st);
    case 19: return run_fourstep<9, 10, IO, false>(a, N, scratch, st);
    case 20: return run_fourstep<10, 10, IO, false>(a, N, scratch, st);
    case 21: return run_fourstep<10, 11, IO, false>(a, N, scratch, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t dispatch_fourstep_circ_f32(int log2m, const FourStepArgs& a, int N, float2* scratch,
                                          cudaStream_t st);
hyena_status_t dispatch_fourstep_circ_bf16(int log2m, const FourStepArgs& a, int N, float2* scratch,
                                           cudaStream_t st);
hyena_status_t dispatch_fourstep_rfft_circ(int log2m, const float* h, int rows, float2* H, float2* scratch,
                                           cudaStream_t st);

}  // namespace hyena
