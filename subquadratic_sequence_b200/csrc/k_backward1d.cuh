// k_backward1d.cuh -- launchers of the 1-D backward pass, included by one
// .cu file per activation type.
#pragma once

#include "backward1d.cuh"
#include "launch.cuh"

namespace hyena {

// Batch slices of the backward: the D S units (G a CTA) run in rounds of
// the resident groups, each unit walking ceil(B / S) sequences; the S in
// [1, smax] of the fewest sequence-rounds (ties: the fewest slices).  On
// 148 SMs c1 (D = 768, B = 8, one CTA of 6 groups an SM) takes S = 8: 7
// rounds of one sequence instead of one round of eight on 128 of the SMs.
template <typename K>
hyena_status_t backward_slices(K kernel, int threads, size_t smem, int G, int B, int D, int smax, int* S)
{
    int sms = 1, occ = 1;
    hyena_status_t st = sm_count(&sms);
    if (st != HYENA_OK) return st;
    cudaError_t e = allow_smem(kernel, smem);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem);
    if (e != cudaSuccess) return from_cuda(e);
    const long slots = (long)sms * (occ < 1 ? 1 : occ) * G;
    long best_cost = -1;
    *S = 1;
    for (int s = 1; s <= smax; ++s) {
        const long rounds = ((long)D * s + slots - 1) / slots;
        const long cost = rounds * ((B + s - 1) / s);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            *S = s;
        }
    }
    return HYENA_OK;
}

// a.S on entry: the most slices the workspace holds
template <int LOG2M, typename IO, bool PS, bool PAD>
hyena_status_t launch_backward(Backward1dArgs a, cudaStream_t st)
{
    using F = Fft1d<LOG2M, PAD>;
    auto kernel = backward1d_kernel<LOG2M, IO, PS, PAD>;
    hyena_status_t s = backward_slices(kernel, F::THREADS, F::SMEM_BYTES, F::G, a.B, a.D, a.S, &a.S);
    if (s != HYENA_OK) return s;
    s = launch(kernel, (unsigned)(((long)a.D * a.S + F::G - 1) / F::G), F::THREADS, F::SMEM_BYTES, st, a);
    if (s != HYENA_OK) return s;
    const int rows = a.N * a.D;
    return launch(dh_finalize_kernel<LOG2M, PS, PAD>, (unsigned)((rows + F::G - 1) / F::G), F::THREADS,
                  F::SMEM_BYTES_FFT, st, a);
}

// PS: a spectrum set per sample (per-sample dh); PAD false: circular mode
// (log2m = log2(L/2) up to 13)
template <typename IO, bool PS = false, bool PAD = true>
hyena_status_t dispatch_backward(int log2m, const Backward1dArgs& a, cudaStream_t st)
{
    switch (log2m) {
    case 4: return launch_backward<4, IO, PS, PAD>(a, st);
    case 5: return launch_backward<5, IO, PS, PAD>(a, st);
    case 6: return launch_backward<6, IO, PS, PAD>(a, st);
    case 7: return launch_backward<7, IO, PS, PAD>(a, st);
    case 8: return launch_backward<8, IO, PS, PAD>(a, st);
    case 9: return launch_backward<9, IO, PS, PAD>(a, st);
    case 10: return launch_backward<10, IO, PS, PAD>(a, st);
    case 11: return launch_backward<11, IO, PS, PAD>(a, st);
    case 12: return launch_backward<12, IO, PS, PAD>(a, st);
    case 13: return launch_backward<13, IO, PS, PAD>(a, st);
    case 14:
        if constexpr (PAD) return launch_backward<14, IO, PS, PAD>(a, st);
        return HYENA_ERR_UNSUPPORTED;
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

}  // namespace hyena
