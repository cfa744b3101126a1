// One FFT level measured on the FP32 pipes and on the tensor cores
// (hyena_dft32_stage).
#include <stdint.h>

#include "dft_stage.cuh"
#include "launch.cuh"

namespace hyena {
int dft_stage_fault_count()
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dft_fault, sizeof(int)) != cudaSuccess) return -1;
    return v;
}
}  // namespace hyena

using namespace hyena;

extern "C" hyena_status_t hyena_dft32_stage(const float* x, float* y, long count, int reps, int method,
                                           void* stream)
{
    if (!x || !y || count < 1 || reps < 1 || (method != 0 && method != 1)) return HYENA_ERR_INVALID_ARG;
    if (((uintptr_t)x % 16) || ((uintptr_t)y % 16)) return HYENA_ERR_INVALID_ARG;
    if (count > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    const size_t bytes = (size_t)count * 32 * sizeof(float2);
    const uintptr_t x0 = (uintptr_t)x, y0 = (uintptr_t)y;
    if (x0 < y0 + bytes && y0 < x0 + bytes) return HYENA_ERR_INVALID_ARG;
    DftStageArgs a = {};
    a.x = reinterpret_cast<const float2*>(x);
    a.y = reinterpret_cast<float2*>(y);
    a.count = count;
    a.reps = reps;
    cudaStream_t st = (cudaStream_t)stream;
    if (method == 0)
        return launch(dft32_simt_kernel, (unsigned)((count + kDftSimtThreads - 1) / kDftSimtThreads),
                      kDftSimtThreads, 0, st, a);
    int sms = 0;
    hyena_status_t s = sm_count(&sms);
    if (s != HYENA_OK) return s;
    const long tiles = (count + dftc::kM - 1) / dftc::kM;
    const long grid = tiles < 2L * sms ? tiles : 2L * sms;
    return launch(dft32_tc_kernel, (unsigned)grid, dftc::kThreads, dftc::kSmem, st, a);
}
