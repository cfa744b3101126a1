// Implicit filter generation launchers (1-D and 2-D).
#include "filter_head_tc.cuh"
#include "launch.cuh"

namespace hyena {

namespace {

// The layers kernel is persistent: at most `per_sm` CTAs per SM, each
// staging the weights once and walking position tiles.
template <bool TWO_D, int PT>
hyena_status_t launch_layers(const FilterGenArgs& a, long npos, int sms, int per_sm, int B, cudaStream_t st)
{
    const long tiles = (npos + PT - 1) / PT;
    long cap = ((long)sms * per_sm + B - 1) / B;
    if (cap < 1) cap = 1;
    return launch(filter_layers_kernel<TWO_D, PT>, dim3((unsigned)(tiles < cap ? tiles : cap), 1, B),
                  kFgThreads, LayerTile<PT>::SMEM, st, a);
}

}  // namespace

// B samples (grid.z) of per-sample filters; B = 1 for shared filters
template <bool TWO_D>
hyena_status_t filter_gen_launches(const FilterGenArgs& a, long npos, int B, cudaStream_t st)
{
    const unsigned ptiles = (unsigned)((npos + kFgTile - 1) / kFgTile);
    if (a.rows <= kFfnWidth)
        return launch(filter_gen_kernel<TWO_D>, dim3(ptiles, 1, B), kFgThreads, kFgFusedSmemBytes, st, a);
    int sms = 0;
    hyena_status_t s = sm_count(&sms);
    if (s != HYENA_OK) return s;
    // short filters: 16-position tiles, so that every SM gets work
    s = (long)ptiles * B >= 2L * sms ? launch_layers<TWO_D, kFgTile>(a, npos, sms, 2, B, st)
                                     : launch_layers<TWO_D, kFgSmallTile>(a, npos, sms, 3, B, st);
    const int head_rows = a.rows - kFfnWidth;
    const unsigned rtiles = (unsigned)((head_rows + kFgRowTile - 1) / kFgRowTile);
    const unsigned ptiles2 = (unsigned)((npos + 127) / 128);
    if (s == HYENA_OK && head_rows > 0 && a.vec) {
        // the tensor-core head: 256 rows per CTA, persistent over 128-position tiles
        const unsigned rt = (unsigned)((head_rows + tch::kN - 1) / tch::kN);
        const long per = (long)sms / ((long)rt * B);
        const unsigned px = (unsigned)(ptiles2 < (per < 1 ? 1 : per) ? ptiles2 : (per < 1 ? 1 : per));
        s = launch(filter_head_tc_kernel<TWO_D>, dim3(px, rt, B), tch::kThreads, tch::kSmem, st, a);
    } else if (s == HYENA_OK && head_rows > 0)
        // 128-position tiles (8 x 8 outputs per thread) once they fill every SM twice
        s = (long)ptiles2 * rtiles * B >= 2L * sms
                ? launch(filter_head_kernel<TWO_D, 2>, dim3(ptiles2, rtiles, B), kFgThreads,
                         fg_head_smem_bytes<2>(), st, a)
                : launch(filter_head_kernel<TWO_D, 1>, dim3(ptiles, rtiles, B), kFgThreads,
                         fg_head_smem_bytes<1>(), st, a);
    // the tail in 16-position tiles unless 64-position tiles fill every SM
    if (s == HYENA_OK)
        s = (long)ptiles * B >= sms
                ? launch(filter_tail_kernel<TWO_D>, dim3(ptiles, 1, B), kFgThreads, kFgTailSmemBytes, st, a)
                : launch(filter_tail16_kernel<TWO_D>,
                         dim3((unsigned)((npos + kFgSmallTile - 1) / kFgSmallTile), 1, B), kFgThreads,
                         kFgTail16SmemBytes, st, a);
    return s;
}

hyena_status_t launch_filter_gen(const FilterGenArgs& a, bool two_d, long npos, int B, cudaStream_t st)
{
    return two_d ? filter_gen_launches<true>(a, npos, B, st) : filter_gen_launches<false>(a, npos, B, st);
}

}  // namespace hyena

extern "C" int hyena_device_fault_count(void)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, hyena::g_tc_fault, sizeof(int)) != cudaSuccess) return -1;
    const int w = hyena::dft_stage_fault_count();
    return w < 0 ? -1 : v + w;
}
