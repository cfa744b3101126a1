// Implicit filter generation launchers (1-D and 2-D).
#include "launch.cuh"

namespace hyena {

template <bool TWO_D>
hyena_status_t filter_gen_launches(const FilterGenArgs& a, long npos, cudaStream_t st)
{
    const unsigned ptiles = (unsigned)((npos + kFgTile - 1) / kFgTile);
    if (a.rows < kFfnWidth + 1)
        return launch(filter_gen_kernel<TWO_D>, dim3(ptiles), kFgThreads, kFgFusedSmemBytes, st, a);
    hyena_status_t s = launch(filter_layers_kernel<TWO_D>,
                              dim3((unsigned)((npos + kFgLayerPos - 1) / kFgLayerPos)), kFgThreads,
                              kFgLayerSmemBytes, st, a);
    const int head_rows = a.rows - kFfnWidth;
    if (s == HYENA_OK)
        s = launch(filter_head_kernel<TWO_D>,
                   dim3(ptiles, (unsigned)((head_rows + kFgRowTile - 1) / kFgRowTile)), kFgThreads,
                   kFgHeadSmemBytes, st, a);
    if (s == HYENA_OK)
        s = launch(filter_tail_kernel<TWO_D>, dim3((unsigned)((npos + kFgTailPos - 1) / kFgTailPos)),
                   kFgThreads, kFgTailSmemBytes, st, a);
    return s;
}

hyena_status_t launch_filter_gen(const FilterGenArgs& a, bool two_d, long npos, cudaStream_t st)
{
    return two_d ? filter_gen_launches<true>(a, npos, st) : filter_gen_launches<false>(a, npos, st);
}

}  // namespace hyena
