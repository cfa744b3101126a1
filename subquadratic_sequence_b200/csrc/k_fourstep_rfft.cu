// Filter spectra for L > 16384: forward columns from h, then forward rows
// with the real split written in the packed layout, wave by wave (PAD
// false: circular mode, the unpadded filters).
#include "k_fourstep.cuh"

namespace hyena {

template <int LM1, int LM2, bool PAD = true>
hyena_status_t run_fourstep_rfft(const float* h, int rows, float2* H, float2* scratch,
                                 cudaStream_t st)
{
    using FS = FourStep<LM1, LM2>;
    FourStepArgs a = {};
    a.v = h;
    a.Hout = H;
    a.S = scratch;
    a.B = 1;
    a.D = rows;
    const long per = wave_seqs(rows, FS::M);
    for (long q0 = 0; q0 < rows; q0 += per) {
        const unsigned nq = (unsigned)(rows - q0 < per ? rows - q0 : per);
        a.q0 = (int)q0;
        hyena_status_t s = launch(fourstep_col_kernel<LM1, LM2, float, 0, PAD>, nq * FS::COL_CTAS_PER_SEQ,
                                  FS::COL_THREADS, FS::COL_SMEM, st, a);
        if (s == HYENA_OK)
            s = launch(fourstep_row_kernel<LM1, LM2, true>, nq * FS::ROW_CTAS_PER_SEQ,
                       FS::ROW_THREADS, FS::ROW_SMEM, st, a);
        if (s != HYENA_OK) return s;
    }
    return HYENA_OK;
}

hyena_status_t dispatch_fourstep_rfft(int log2m, const float* h, int rows, float2* H,
                                      float2* scratch, cudaStream_t st)
{
    switch (log2m) {
    case 15: return run_fourstep_rfft<7, 8>(h, rows, H, scratch, st);
    case 16: return run_fourstep_rfft<8, 8>(h, rows, H, scratch, st);
    case 17: return run_fourstep_rfft<8, 9>(h, rows, H, scratch, st);
    case 18: return run_fourstep_rfft<9, 9>(h, rows, H, scratch, st);
    case 19: return run_fourstep_rfft<9, 10>(h, rows, H, scratch, st);
    case 20: return run_fourstep_rfft<10, 10>(h, rows, H, scratch, st);
    case 21: return run_fourstep_rfft<10, 11>(h, rows, H, scratch, st);
    case 22: return run_fourstep_rfft<11, 11>(h, rows, H, scratch, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

// circular mode: log2m = log2(L/2)
hyena_status_t dispatch_fourstep_rfft_circ(int log2m, const float* h, int rows, float2* H, float2* scratch,
                                           cudaStream_t st)
{
    switch (log2m) {
    case 14: return run_fourstep_rfft<7, 7, false>(h, rows, H, scratch, st);
    case 15: return run_fourstep_rfft<7, 8, false>(h, rows, H, scratch, st);
    case 16: return run_fourstep_rfft<8, 8, false>(h, rows, H, scratch, st);
    case 17: return run_fourstep_rfft<8, 9, false>(h, rows, H, scratch, st);
    case 18: return run_fourstep_rfft<9, 9, false>(h, rows, H, scratch, st);
    case 19: return run_fourstep_rfft<9, 10, false>(h, rows, H, scratch, st);
    case 20: return run_fourstep_rfft<10, 10, false>(h, rows, H, scratch, st);
    case 21: return run_fourstep_rfft<10, 11, false>(h, rows, H, scratch, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
