// k_fourstep_bwd.cuh -- launch sequence of the four-step backward, included
// by one .cu file per activation type.
#pragma once

#include "fourstep_bwd.cuh"
#include "launch.cuh"

namespace hyena {

// sequences a wave of the four-step backward holds (the forward's scratch budget)
inline long bwd_wave_cap(long M) { return wave_seqs(1L << 30, M); }

// Workspace layout of the four-step backward (bytes): acc [sets][N][D][M]
// (sets = B with per-sample spectra, else 1), zsave [N][wcap][M1][RS],
// csave [N][wcap][M/2], scratch [wcap][M].
struct FourStepBwdLayout {
    size_t acc, zsave, csave, scratch, total;
    long wcap;
};

// circular: c_n of M value pairs a sequence (else M/2)
template <int LM1, int LM2>
FourStepBwdLayout fourstep_bwd_layout_n(int D, int N, int sets, bool circular = false)
{
    using FS = FourStep<LM1, LM2>;
    auto up = [](size_t n) { return (n + 255) / 256 * 256; };
    FourStepBwdLayout l;
    l.wcap = bwd_wave_cap(FS::M);
    l.acc = 0;
    l.zsave = l.acc + up(sizeof(float2) * (size_t)sets * N * D * FS::M);
    l.csave = l.zsave + up(sizeof(float2) * (size_t)N * l.wcap * FS::M1 * FS::ROW_STRIDE);
    l.scratch = l.csave + up(sizeof(float2) * (size_t)N * l.wcap * (circular ? FS::M : FS::M / 2));
    l.total = l.scratch + up(sizeof(float2) * (size_t)l.wcap * FS::M);
    return l;
}

template <int LM1, int LM2, typename IO, bool PAD = true>
hyena_status_t run_fourstep_bwd(FourStepBwdArgs a, int N, cudaStream_t st)
{
    using FS = FourStep<LM1, LM2>;
    using FB = FourStepBwd<LM1, LM2>;
    FourStepArgs& f = a.f;
    const long nseq = (long)f.B * f.D, per = a.wcap;
    const long sets = f.H_bstride != 0 ? f.B : 1;             // dh spectra per (n, d)
    f.n_last = N - 1;
    const cudaError_t e = cudaMemsetAsync(a.acc, 0, sizeof(float2) * (size_t)sets * N * f.D * FS::M, st);
    if (e != cudaSuccess) return from_cuda(e);
    for (long q0 = 0; q0 < nseq; q0 += per) {
        const unsigned nq = (unsigned)(nseq - q0 < per ? nseq - q0 : per);
        f.q0 = (int)q0;
        f.n = 0;
        a.nq = (int)nq;
        // A: the forward, saving Zc and c_n
        hyena_status_t s = launch(fourstep_col_kernel<LM1, LM2, IO, 0, PAD>, nq * FS::COL_CTAS_PER_SEQ,
                                  FS::COL_THREADS, FS::COL_SMEM, st, f);
        for (int n = 0; n < N && s == HYENA_OK; ++n) {
            f.n = n;
            a.last = n + 1 == N;
            s = launch(fourstep_bwd_row_kernel<LM1, LM2, 0>, nq * FS::ROW_CTAS_PER_SEQ, FS::ROW_THREADS,
                       FS::ROW_SMEM, st, a);
            if (s == HYENA_OK)
                s = launch(fourstep_bwd_col_kernel<LM1, LM2, IO, 0, PAD>, nq * FS::COL_CTAS_PER_SEQ,
                           FS::COL_THREADS, FS::COL_SMEM, st, a);
        }
        // B: the orders in reverse; the rows per channel of the wave
        const unsigned nch = (unsigned)((q0 + nq - 1) / f.B - q0 / f.B + 1);
        for (int n = N - 1; n >= 0 && s == HYENA_OK; --n) {
            f.n = n;
            a.first = n == N - 1;
            s = launch(fourstep_bwd_col_kernel<LM1, LM2, IO, 1, PAD>, nq * FS::COL_CTAS_PER_SEQ, FS::COL_THREADS,
                       FS::COL_SMEM, st, a);
            if (s == HYENA_OK)
                s = launch(fourstep_bwd_row_kernel<LM1, LM2, 1>, nch * FS::ROW_CTAS_PER_SEQ, FS::ROW_THREADS,
                           FB::ROW_SMEM_B, st, a);
        }
        if (s == HYENA_OK)
            s = launch(fourstep_bwd_col_kernel<LM1, LM2, IO, 2, PAD>, nq * FS::COL_CTAS_PER_SEQ, FS::COL_THREADS,
                       FS::COL_SMEM, st, a);
        if (s != HYENA_OK) return s;
    }
    // dh_n, db_n from the sets*N*D accumulated spectra, a wave of rows at a time
    const long rows = sets * N * f.D;
    for (long r0 = 0; r0 < rows; r0 += per) {
        const unsigned nq = (unsigned)(rows - r0 < per ? rows - r0 : per);
        f.q0 = (int)r0;
        a.nq = (int)nq;
        hyena_status_t s = launch(fourstep_bwd_row_kernel<LM1, LM2, 2>, nq * FS::ROW_CTAS_PER_SEQ,
                                  FS::ROW_THREADS, FS::ROW_SMEM, st, a);
        if (s == HYENA_OK)
            s = launch(fourstep_bwd_col_kernel<LM1, LM2, IO, 3, PAD>, nq * FS::COL_CTAS_PER_SEQ, FS::COL_THREADS,
                       FS::COL_SMEM, st, a);
        if (s != HYENA_OK) return s;
    }
    if (f.H_bstride != 0) {          // per-sample: db from the B lag-0 values (any B)
        const int nd = N * f.D;
        // dh rows of L floats: L = M (padded), 2M (circular)
        return launch(dbias_sum_kernel<PAD ? FS::M : 2 * FS::M>, (unsigned)((nd + 255) / 256), 256, 0, st, a);
    }
    return HYENA_OK;
}

template <typename IO>
hyena_status_t dispatch_fourstep_bwd(int log2m, const FourStepBwdArgs& a, int N, cudaStream_t st)
{
    switch (log2m) {
    case 15: return run_fourstep_bwd<7, 8, IO>(a, N, st);
    case 16: return run_fourstep_bwd<8, 8, IO>(a, N, st);
    case 17: return run_fourstep_bwd<8, 9, IO>(a, N, st);
    case 18: return run_fourstep_bwd<8, 10, IO>(a, N, st);
    case 19: return run_fourstep_bwd<9, 10, IO>(a, N, st);
    case 20: return run_fourstep_bwd<10, 10, IO>(a, N, st);
    case 21: return run_fourstep_bwd<10, 11, IO>(a, N, st);
    case 22: return run_fourstep_bwd<11, 11, IO>(a, N, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

inline FourStepBwdLayout fourstep_bwd_layout(int log2m, int D, int N, int sets = 1, bool circular = false)
{
    switch (log2m) {
    case 14: return fourstep_bwd_layout_n<7, 7>(D, N, sets, circular);
    case 15: return fourstep_bwd_layout_n<7, 8>(D, N, sets, circular);
    case 16: return fourstep_bwd_layout_n<8, 8>(D, N, sets, circular);
    case 17: return fourstep_bwd_layout_n<8, 9>(D, N, sets, circular);
    case 18: return fourstep_bwd_layout_n<8, 10>(D, N, sets, circular);
    case 19: return fourstep_bwd_layout_n<9, 10>(D, N, sets, circular);
    case 20: return fourstep_bwd_layout_n<10, 10>(D, N, sets, circular);
    case 21: return fourstep_bwd_layout_n<10, 11>(D, N, sets, circular);
    default: return fourstep_bwd_layout_n<11, 11>(D, N, sets, circular);
    }
}

// circular mode: log2m = log2(L/2), 14 .. 21 (16384 < L <= 2^22)
template <typename IO>
hyena_status_t dispatch_fourstep_bwd_circ(int log2m, const FourStepBwdArgs& a, int N, cudaStream_t st)
{
    switch (log2m) {
    case 14: return run_fourstep_bwd<7, 7, IO, false>(a, N, st);
    case 15: return run_fourstep_bwd<7, 8, IO, false>(a, N, st);
    case 16: return run_fourstep_bwd<8, 8, IO, false>(a, N, st);
    case 17: return run_fourstep_bwd<8, 9, IO, false>(a, N, st);
    case 18: return run_fourstep_bwd<8, 10, IO, false>(a, N, st);
    case 19: return run_fourstep_bwd<9, 10, IO, false>(a, N, st);
    case 20: return run_fourstep_bwd<10, 10, IO, false>(a, N, st);
    case 21: return run_fourstep_bwd<10, 11, IO, false>(a, N, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t dispatch_fourstep_bwd_f32(int log2m, const FourStepBwdArgs& a, int N, cudaStream_t st);
hyena_status_t dispatch_fourstep_bwd_bf16(int log2m, const FourStepBwdArgs& a, int N, cudaStream_t st);
hyena_status_t dispatch_fourstep_bwd_circ_f32(int log2m, const FourStepBwdArgs& a, int N, cudaStream_t st);
hyena_status_t dispatch_fourstep_bwd_circ_bf16(int log2m, const FourStepBwdArgs& a, int N, cudaStream_t st);

}  // namespace hyena
