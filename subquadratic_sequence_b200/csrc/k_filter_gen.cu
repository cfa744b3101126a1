// Implicit filter generation launchers (1-D and 2-D).
#include "launch.cuh"

namespace hyena {

hyena_status_t launch_filter_gen(const FilterGenArgs& a, bool two_d, long npos, cudaStream_t st)
{
    const dim3 grid((unsigned)((npos + kFgTile - 1) / kFgTile),
                    (unsigned)((a.rows + kFgRowTile - 1) / kFgRowTile));
    return two_d ? launch(filter_gen_kernel<true>, grid, kFgThreads, kFgSmemBytes, st, a)
                 : launch(filter_gen_kernel<false>, grid, kFgThreads, kFgSmemBytes, st, a);
}

}  // namespace hyena
