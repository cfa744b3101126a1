// dft_stage.cuh -- one FFT level computed two ways, to measure which
// arithmetic units suit the path's FFTs on sm_100a.
//
// "Long Context Language Models ... #690" (7:06) notes that GPUs are built
// for matrix multiplication and that FFT convolutions can be recast as
// matrix products (the FlashFFTConv idea).  The long-sequence FFTs here are
// made of radix-32 levels (1024 = 32 x 32 points per row or column), so the
// measured unit is a batch of independent 32-point complex DFTs, each
// applied `reps` times in a row to its previous result with the unitary
// scale 1/sqrt(32) (four applications give the input back):
//  SIMT     one thread per vector: dft<32> in registers, then every value
//           through shared memory and back with a barrier, as a pass of the
//           shared-memory FFTs exchanges its data;
//  tcgen05  128 vectors per tile as a 128 x 64 real matrix (re, im
//           interleaved) times the 64 x 64 real form of the scaled DFT
//           matrix, in TF32 with the hi/lo split for float32 accuracy (three
//           MMAs per K step), the accumulator in tensor memory; each
//           repetition reads it back, splits it and writes it to shared
//           memory as the next operand, the round trip a level of a
//           tensor-core FFT needs.
// Both read x once and write y once, so with many repetitions the time per
// repetition is the cost of one FFT level on that unit.
#pragma once

#include "hyena_common.cuh"
#include "tcgen05.cuh"

namespace hyena {

struct DftStageArgs {
    const float2* x;               // [count][32] complex
    float2* y;                     // [count][32] complex
    long count;
    int reps;
};

// set when a tensor-core wait timed out (read by hyena_device_fault_count);
// this header is included by one translation unit only
static __device__ int g_dft_fault;

constexpr int kDftSimtThreads = 128;

__global__ void __launch_bounds__(kDftSimtThreads) dft32_simt_kernel(DftStageArgs a)
{
    grid_dependency_begin();
    constexpr int T = kDftSimtThreads;
    __shared__ float2 sm[padded_size(32 * T)];
    const int t = threadIdx.x;
    const long v = (long)blockIdx.x * T + t;
    const bool active = v < a.count;
    const long vv = active ? v : a.count - 1;
    constexpr float scale = 0.17677669529663688f;           // 1/sqrt(32)
    float2 r[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __ldg(a.x + vv * 32 + i);
    for (int rep = 0; rep < a.reps; ++rep) {
        dft<32, -1>(r);
#pragma unroll
        for (int i = 0; i < 32; ++i) sm[pad16(i * T + t)] = make_float2(r[i].x * scale, r[i].y * scale);
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = sm[pad16(i * T + t)];
        __syncthreads();
    }
    if (active)
#pragma unroll
        for (int i = 0; i < 32; ++i) a.y[v * 32 + i] = r[i];
}

namespace dftc {
constexpr int kM = 128;            // vectors per tile
constexpr int kK = 64;             // input reals per vector
constexpr int kN = 64;             // output reals per vector
constexpr int kThreads = 128;
constexpr int kTmemCols = 64;
constexpr size_t kSmem = 2 * (size_t)kM * kK * 4 + 2 * (size_t)kN * kK * 4 + 64;
// word offset of the 4-real chunk c of row n in the K-major no-swizzle layout
__device__ __forceinline__ int chunk_off(int n, int c) { return (n >> 3) * 512 + c * 32 + (n & 7) * 4; }
}  // namespace dftc

__global__ void __launch_bounds__(dftc::kThreads, 2) dft32_tc_kernel(DftStageArgs a)
{
    using namespace dftc;
    using namespace tc5;
    grid_dependency_begin();
    extern __shared__ __align__(1024) unsigned char dft_smem[];
    uint32_t* sAhi = reinterpret_cast<uint32_t*>(dft_smem);
    uint32_t* sAlo = sAhi + kM * kK;
    uint32_t* sBhi = sAlo + kM * kK;
    uint32_t* sBlo = sBhi + kN * kK;
    uint64_t* sBar = reinterpret_cast<uint64_t*>(sBlo + kN * kK);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sBar + 1);
    int* sFault = reinterpret_cast<int*>(sTmem + 1);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

    // B: row 2k (re of output k) = [cos, sin] per input n, row 2k + 1 (im)
    // = [-sin, cos], angle 2 pi k n / 32, scaled by 1/sqrt(32)
    for (int e = tid; e < kN * (kK / 4); e += kThreads) {
        const int o = e / (kK / 4), c = e % (kK / 4);
        const int k = o >> 1;
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int n = 2 * c + i;
            float sn, cs;
            sincospif((float)((k * n) % 32) / 16.0f, &sn, &cs);
            cs *= 0.17677669529663688f;
            sn *= 0.17677669529663688f;
            const float w0 = (o & 1) ? -sn : cs, w1 = (o & 1) ? cs : sn;
            split_tf32(w0, hi[2 * i], lo[2 * i]);
            split_tf32(w1, hi[2 * i + 1], lo[2 * i + 1]);
        }
        *reinterpret_cast<uint4*>(sBhi + chunk_off(o, c)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sBlo + chunk_off(o, c)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    if (tid == 0) {
        mbar_init(sBar);
        *sFault = 0;
    }
    if (warp == 0) tmem_alloc(sTmem, kTmemCols);
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *sTmem, bar = smem_u32(sBar);
    const uint32_t idesc = instr_desc_tf32(kN);
    const long ntiles = (a.count + kM - 1) / kM;
    uint32_t phase = 0;

    for (long tile = blockIdx.x; tile < ntiles && !*sFault; tile += gridDim.x) {
        // thread tid holds vector m = tid of the tile: 32 complex = 16 chunks
        const long v = tile * kM + tid;
        const bool active = v < a.count;
        float r[kK];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float2 z = active ? __ldg(a.x + v * 32 + i) : make_float2(0.0f, 0.0f);
            r[2 * i] = z.x;
            r[2 * i + 1] = z.y;
        }
        for (int rep = 0; rep < a.reps; ++rep) {
#pragma unroll
            for (int c = 0; c < kK / 4; ++c) {
                uint4 hi, lo;
                split_tf32(r[4 * c], hi.x, lo.x);
                split_tf32(r[4 * c + 1], hi.y, lo.y);
                split_tf32(r[4 * c + 2], hi.z, lo.z);
                split_tf32(r[4 * c + 3], hi.w, lo.w);
                *reinterpret_cast<uint4*>(sAhi + chunk_off(tid, c)) = hi;
                *reinterpret_cast<uint4*>(sAlo + chunk_off(tid, c)) = lo;
            }
            fence_async_smem();
            __syncthreads();
            if (tid == 0) {
                fence_after();
                const uint32_t ahi = smem_u32(sAhi), alo = smem_u32(sAlo), bhi = smem_u32(sBhi),
                               blo = smem_u32(sBlo);
#pragma unroll
                for (int s = 0; s < kK / 8; ++s) {
                    mma_tf32(tmem, smem_desc(alo + 256 * s, 128, 2048), smem_desc(bhi + 256 * s, 128, 2048), idesc,
                             s > 0);
                    mma_tf32(tmem, smem_desc(ahi + 256 * s, 128, 2048), smem_desc(blo + 256 * s, 128, 2048), idesc,
                             1);
                    mma_tf32(tmem, smem_desc(ahi + 256 * s, 128, 2048), smem_desc(bhi + 256 * s, 128, 2048), idesc,
                             1);
                }
                mma_commit(bar);
            }
            if (!mbar_wait_bounded(bar, phase)) *sFault = 1;
            phase ^= 1;
            __syncthreads();
            if (*sFault) break;
            fence_after();
            // accumulator lanes 32 warp .. (= this thread's vector), 64 columns
#pragma unroll
            for (int q = 0; q < kN / 16; ++q) tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + 16 * q, r + 16 * q);
            fence_before();
            __syncthreads();
        }
        if (active && !*sFault)
#pragma unroll
            for (int i = 0; i < 32; ++i) a.y[v * 32 + i] = make_float2(r[2 * i], r[2 * i + 1]);
    }
    if (*sFault && tid == 0) atomicExch(&g_dft_fault, 1);
    fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace hyena
