// filter_head_tc.cuh -- the head of the implicit filter network on the
// fifth-generation tensor cores (tcgen05: operands in shared memory,
// accumulator in tensor memory).
//
// The head is the one dense contraction of the path: h[r][p] = window(r, p)
// * sum_j Wout[r][j] a3[j][p] over the 64 units of the last sine layer
// ("Long Context Language Models ... #690", 4:29: the filter is produced by
// an MLP from the position), a [rows x 64] x [64 x positions] product.  Each
// CTA keeps up to 256 rows of Wout in shared memory and walks tiles of 128
// positions: the 128 x 64 tile of a3 (read from the stash rows of h) goes
// to shared memory, one thread issues the MMAs (M = 128 positions, N = the
// rows, K = 64 in steps of 8), and the sixteen warps read the 128 x N fp32
// accumulator back from tensor memory, apply the window and store h.
//
// Float32 accuracy with TF32 products: each operand is split as
// x = hi + lo with hi = tf32(x) and lo = tf32(x - hi) (both rounded to
// nearest), and D = A_lo B_hi + A_hi B_lo + A_hi B_hi accumulates in fp32
// (the dropped A_lo B_lo and the operands' residuals are below 2^-21 of the
// product), so the filters stay within the float32 tolerance of the SIMT
// head.
//
// Shared-memory operand layouts: both operands K-major, no swizzle (the
// canonical tcgen05 layout of 8-row x 16-byte core matrices): the 16-byte
// chunk of row n (a position for A, a row of h for B) and units 4c..4c+3
// sits at (n/8)*2048 + c*128 + (n%8)*16 bytes, so one MMA's K = 8 units
// are two chunks 128 bytes apart (leading byte offset) and row groups are
// 2048 bytes apart (stride byte offset).  A warp writes 32 consecutive
// positions of one chunk: four 128-byte runs, the minimum four wavefronts.
// Every wait on the tensor cores is bounded: after about two seconds the
// kernel records a fault (hyena_device_fault_count), frees its tensor
// memory and returns.
#pragma once

#include "filter_gen.cuh"
#include "tcgen05.cuh"

namespace hyena {

// set when a tensor-core wait timed out (read by hyena_device_fault_count);
// this header is included by one translation unit only
static __device__ int g_tc_fault;

namespace tch {
constexpr int kM = 128;                 // positions per tile
constexpr int kN = 256;                 // rows per CTA, at most
constexpr int kK = kFfnWidth;           // 64 units
constexpr int kThreads = 512;             // 16 warps: four per accumulator lane group
constexpr int kTmemCols = 512;        // two accumulators of 256 columns
constexpr int kBBytes = kN * kK * 4;    // 64 KB per split half
constexpr int kABytes = kM * kK * 4;    // 32 KB per split half
constexpr size_t kSmem = 2 * (size_t)kBBytes + 2 * (size_t)kABytes + 4 * kN + 64;
static_assert(kSmem <= 227 * 1024, "shared memory");

}  // namespace tch

// Rows r0 .. r0 + 255 (grid.y) of the head, all position tiles
// blockIdx.x, blockIdx.x + gridDim.x, ...; a.vec must hold (positions a
// multiple of 4, h 16-byte aligned).
template <bool TWO_D>
__global__ void __launch_bounds__(tch::kThreads, 1) filter_head_tc_kernel(FilterGenArgs a)
{
    using namespace tch;
    using namespace tc5;
    grid_dependency_begin();
    select_sample(a);
    extern __shared__ __align__(1024) unsigned char tc_smem[];
    uint32_t* sBhi = reinterpret_cast<uint32_t*>(tc_smem);
    uint32_t* sBlo = sBhi + kN * kK;
    uint32_t* sAhi = sBlo + kN * kK;
    uint32_t* sAlo = sAhi + kM * kK;
    float* sC = reinterpret_cast<float*>(sAlo + kM * kK);      // window coefficients (log2 units)
    uint64_t* sBar = reinterpret_cast<uint64_t*>(sC + kN);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sBar + 1);
    int* sFault = reinterpret_cast<int*>(sTmem + 1);

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const long npos = fg_positions<TWO_D>(a);
    const int stash_row = a.rows - kFfnWidth;
    const int r0 = blockIdx.y * kN;
    const int nrows = min(kN, stash_row - r0);
    const int N = (nrows + 15) & ~15;                       // MMA N: a multiple of 16
    const float* stash = a.h + (long)stash_row * npos;

    // Wout rows r0 .. r0 + N - 1, split, K-major; window coefficients
    for (int e = tid; e < kN * (kK / 4); e += kThreads) {
        const int n = e / (kK / 4), c = e % (kK / 4);
        uint32_t hi[4] = {0, 0, 0, 0}, lo[4] = {0, 0, 0, 0};
        if (n < nrows) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int j = 4 * c + i;
                const float w = j < a.width ? __ldg(a.Wout + (long)(r0 + n) * a.width + j) : 0.0f;
                split_tf32(w, hi[i], lo[i]);
            }
        }
        const int off = ((n >> 3) * 512 + c * 32 + (n & 7) * 4);   // in 4-byte words
        *reinterpret_cast<uint4*>(sBhi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sBlo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    for (int n = tid; n < kN; n += kThreads)
        sC[n] = n < nrows ? window_coeff(a, __ldg(a.alpha + (r0 + n) % a.D)) * 1.4426950408889634f : 0.0f;
    if (tid == 0) {
        mbar_init(sBar);
        *sFault = 0;
    }
    if (warp == 0) tmem_alloc(sTmem, kTmemCols);
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t bar = smem_u32(sBar);
    const uint32_t idesc = instr_desc_tf32(N);
    const long ntiles = (npos + kM - 1) / kM;
    uint32_t phase = 0;

    // thread (chunk c = e / 128, position m = e % 128, e = tid + 512 i) holds
    // units 4c..4c+3 of position p0 + m (a warp: 32 consecutive positions);
    // the next tile's values are loaded while this tile's MMAs and
    // epilogue run
    constexpr int kPer = kM * (kK / 4) / kThreads;           // 4 chunks per thread
    float4 nxt[kPer];
    auto load_tile = [&](long tile) {
        const long p0 = tile * kM;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = tid + kThreads * i, c = e / kM, m = e % kM;
            const long p = p0 + m;
            float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (tile < ntiles && p < npos) {
                const float* q = stash + (long)(4 * c) * npos + p;
                v = make_float4(__ldg(q), __ldg(q + npos), __ldg(q + 2 * npos), __ldg(q + 3 * npos));
            }
            nxt[i] = v;
        }
    };
    // the 128 x 64 tile in registers -> split into the two K-major operands
    auto stage_tile = [&]() {
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = tid + kThreads * i, c = e / kM, m = e % kM;
            uint4 hi, lo;
            split_tf32(nxt[i].x, hi.x, lo.x);
            split_tf32(nxt[i].y, hi.y, lo.y);
            split_tf32(nxt[i].z, hi.z, lo.z);
            split_tf32(nxt[i].w, hi.w, lo.w);
            const int off = (m >> 3) * 512 + c * 32 + (m & 7) * 4;     // words
            *reinterpret_cast<uint4*>(sAhi + off) = hi;
            *reinterpret_cast<uint4*>(sAlo + off) = lo;
        }
        fence_async_smem();
        __syncthreads();
    };
    // one thread: D[buf] = A B^T in three split products per K step
    auto issue_mma = [&](int buf) {
        if (tid == 0) {
            fence_after();
            const uint32_t d = tmem + 256 * buf;
            const uint32_t ahi = smem_u32(sAhi), alo = smem_u32(sAlo), bhi = smem_u32(sBhi), blo = smem_u32(sBlo);
#pragma unroll
            for (int s = 0; s < kK / 8; ++s) {
                // units 8s .. 8s + 7: chunks 2s and 2s + 1, at +256 s
                const uint64_t dAhi = smem_desc(ahi + 256 * s, 128, 2048);
                const uint64_t dAlo = smem_desc(alo + 256 * s, 128, 2048);
                const uint64_t dBhi = smem_desc(bhi + 256 * s, 128, 2048);
                const uint64_t dBlo = smem_desc(blo + 256 * s, 128, 2048);
                mma_tf32(d, dAlo, dBhi, idesc, s > 0);
                mma_tf32(d, dAhi, dBlo, idesc, 1);
                mma_tf32(d, dAhi, dBhi, idesc, 1);
            }
            mma_commit(bar);
        }
    };

    // Pipeline over the CTA's tiles t_0, t_1, ...: while the epilogue of t_i
    // reads accumulator i % 2, the MMAs of t_{i+1} fill the other one and the
    // loads of t_{i+2} are in flight.
    load_tile(blockIdx.x);
    if (blockIdx.x < ntiles) {
        stage_tile();
        issue_mma(0);
    }
    load_tile(blockIdx.x + gridDim.x);
    int it = 0;
    for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        const long p0 = tile * kM;
        if (!mbar_wait_bounded(bar, phase)) *sFault = 1;
        phase ^= 1;
        __syncthreads();
        if (*sFault) break;
        if (tile + gridDim.x < ntiles) {
            stage_tile();                       // A of the next tile: its operand space is free now
            issue_mma((it + 1) & 1);
            load_tile(tile + 2L * gridDim.x);
        }
        fence_after();
        // epilogue: warp w reads accumulator lanes 32 (w % 4) .. (positions)
        // and column chunks of 16 rows c = w / 4, w / 4 + 4, ..., two chunks
        // per wait; the row pointer advances by whole rows
        {
            const int lg = warp & 3;
            const long p = p0 + 32 * lg + lane;
            const float u = window_u<TWO_D>(a, p);
            const bool inside = p < npos;
            const uint32_t base = tmem + 256 * (it & 1) + ((uint32_t)(32 * lg) << 16);
            for (int c0 = warp >> 2; c0 < N / 16; c0 += 8) {
                uint32_t v[2][16];
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    if (c0 + 4 * q < N / 16) tmem_ld16_issue(base + 16 * (c0 + 4 * q), v[q]);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int c = c0 + 4 * q;
                    if (c >= N / 16) break;
                    const float4* cw = reinterpret_cast<const float4*>(sC + 16 * c);
                    float* hp = a.h + (long)(r0 + 16 * c) * npos + p;
#pragma unroll
                    for (int j4 = 0; j4 < 4; ++j4) {
                        const float4 k4 = cw[j4];
                        const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            const int j = 4 * j4 + jj;
                            if (inside && 16 * c + j < nrows) *hp = __uint_as_float(v[q][j]) * exp2f(kk[jj] * u);
                            hp += npos;
                        }
                    }
                }
            }
        }
        fence_before();
        __syncthreads();            // accumulator it % 2 free for the MMAs after next
    }
    if (*sFault && tid == 0) atomicExch(&g_tc_fault, 1);
    fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace hyena
