// launch.cuh -- internal (not exported) launch helpers shared by the
// library's translation units.  Each kernel family is instantiated and
// launched in its own .cu file so the library compiles in parallel;
// hyena_api.cu validates arguments and calls these dispatchers.
#pragma once

#include <cuda_runtime.h>

#include "backward1d.cuh"
#include "filter_gen.cuh"
#include "fourstep.cuh"
#include "fused1d.cuh"
#include "hyena.h"

namespace hyena {

constexpr int kMinLog2 = 4;        // L >= 16
constexpr int kMaxLog2Fused = 14;  // single-CTA path: L <= 16384
constexpr int kMaxLog2 = 22;       // four-step path: L <= 2^22
// the scratch of one wave of long sequences stays under this (L2 resident)
constexpr size_t kWaveScratchBytes = 64u << 20;

// Maps a CUDA error to a status and records it for hyena_last_cuda_error().
hyena_status_t from_cuda(cudaError_t e);

// Opts a kernel in to more than 48 KB of dynamic shared memory.
template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes)
{
    if (bytes <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Launches a kernel (every kernel starts with grid_dependency_begin()).
// With `pdl` it is launched with programmatic stream serialisation, so its
// CTAs may be placed while the previous kernel drains; the 2-D FFT kernels
// measured slower that way and are launched plainly.
template <typename A>
hyena_status_t launch(void (*kernel)(A), dim3 grid, int threads, size_t smem, cudaStream_t st, const A& a,
                      bool pdl = true)
{
    cudaError_t e = allow_smem(kernel, smem);
    if (e != cudaSuccess) return from_cuda(e);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return from_cuda(cudaLaunchKernelEx(&cfg, kernel, a));
}

// Number of SMs of the current device.
inline hyena_status_t sm_count(int* n)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess && *n < 1) *n = 1;
    return from_cuda(e);
}

// sequences per wave of the four-step path (scratch = wave * L complex)
inline long wave_seqs(long nseq, long L)
{
    long per = (long)(kWaveScratchBytes / (sizeof(float2) * (size_t)L));
    if (per < 1) per = 1;
    return nseq < per ? nseq : per;
}

// tensor-core waits of hyena_dft32_stage that timed out (-1: query failed)
int dft_stage_fault_count();
hyena_status_t dispatch_fused_f32(int log2m, const Fused1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_fused_bf16(int log2m, const Fused1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_fused_ps_f32(int log2m, const Fused1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_fused_ps_bf16(int log2m, const Fused1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_rfft(int log2m, const Rfft1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_fourstep_f32(int log2m, const FourStepArgs& a, int N, float2* scratch,
                                     cudaStream_t st);
hyena_status_t dispatch_fourstep_bf16(int log2m, const FourStepArgs& a, int N, float2* scratch,
                                      cudaStream_t st);
hyena_status_t dispatch_fourstep_rfft(int log2m, const float* h, int rows, float2* H,
                                      float2* scratch, cudaStream_t st);
hyena_status_t launch_filter_gen(const FilterGenArgs& a, bool two_d, long npos, int B, cudaStream_t st);
hyena_status_t dispatch_backward_f32(int log2m, const Backward1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_backward_bf16(int log2m, const Backward1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_backward_ps_f32(int log2m, const Backward1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_backward_ps_bf16(int log2m, const Backward1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_backward_circ_f32(int log2m, const Backward1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_backward_circ_bf16(int log2m, const Backward1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_backward_circ_ps_f32(int log2m, const Backward1dArgs& a, cudaStream_t st);
hyena_status_t dispatch_backward_circ_ps_bf16(int log2m, const Backward1dArgs& a, cudaStream_t st);

}  // namespace hyena
