// k_fourstep.cuh -- wave-by-wave launch sequences of the four-step path,
// included by one .cu file per activation type (and one for the spectra).
#pragma once

#include "launch.cuh"

namespace hyena {

// The order-N forward over B*D sequences, wave by wave: per wave one
// column launch (from v), then per order a row launch and a column launch.
template <int LM1, int LM2, typename IO>
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
        hyena_status_t s = launch(fourstep_col_kernel<LM1, LM2, IO, 0>, nq * FS::COL_CTAS_PER_SEQ,
                                  FS::COL_THREADS, FS::COL_SMEM, st, a);
        for (int n = 0; n < N && s == HYENA_OK; ++n) {
            a.n = n;
            s = launch(fourstep_row_kernel<LM1, LM2, false>, nq * FS::ROW_CTAS_PER_SEQ,
                       FS::ROW_THREADS, FS::ROW_SMEM, st, a);
            if (s != HYENA_OK) break;
            s = n + 1 < N ? launch(fourstep_col_kernel<LM1, LM2, IO, 1>, nq * FS::COL_CTAS_PER_SEQ,
                                   FS::COL_THREADS, FS::COL_SMEM, st, a)
                          : launch(fourstep_col_kernel<LM1, LM2, IO, 2>, nq * FS::COL_CTAS_PER_SEQ,
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
    case 18: return run_fourstep<9, 9, IO>(a, N, scratch, st);
    case 19: return run_fourstep<9, 10, IO>(a, N, scratch, st);
    case 20: return run_fourstep<10, 10, IO>(a, N, scratch, st);
    case 21: return run_fourstep<10, 11, IO>(a, N, scratch, st);
    case 22: return run_fourstep<11, 11, IO>(a, N, scratch, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
