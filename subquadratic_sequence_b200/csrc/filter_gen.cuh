// filter_gen.cuh -- implicit filter generation on the GPU.
//
// "Long Context Language Models and their Biological Applications with
// Eric Nguyen - #690" (4:29): the long filter is not stored tap by tap but
// produced by an MLP from the position.  This library's reading of that
// MLP: positional features (1-D: [t, sin 2 pi k t, cos 2 pi k t]_{k=1..K},
// t = i/L; 2-D: [ty, tx, (sin, cos)(2 pi k ty)_k, (sin, cos)(2 pi k tx)_k]),
// three bias-free Linear + sin layers of width <= 64, a bias-free linear
// head to N*D rows (filter n, channel d = row n*D + d), and an exponential
// decay window exp(-alpha_d i / div) (2-D: exp(-alpha_c (iy + ix) / div)
// as the product of the two axis windows).
//
// Three launches, no recomputation:
//  layers: all threads of a CTA evaluate the three sine layers for 16
//          positions (16 threads per position, 4 output units each, weights
//          broadcast from shared memory) and stash a3 [64][positions] in
//          the LAST 64 rows of h (they are outputs too, written last);
//  head:   h[r][p] = (sum_j Wout[r][j] a3[j][p]) * window for the rows
//          before the stash, as 128-row x 64-position tiles out of shared
//          memory, written coalesced along the position;
//  tail:   the head for the 64 stash rows, 16 positions per CTA: each CTA
//          loads its own tile of a3 into shared memory before overwriting it.
// With fewer than 64 head rows the layers are evaluated inside the head
// kernel instead (one launch).
#pragma once

#include "hyena_common.cuh"

namespace hyena {

constexpr int kFfnWidth = 64;      // widths above this are rejected
constexpr int kFfnMaxIn = 66;      // 2 + 4 * 16 bands

struct FilterGenArgs {
    const float *W1, *W2, *W3, *Wout, *alpha;
    int n_in, width, rows;         // rows = N * D
    int D;                         // channels (alpha index = row % D)
    int L;                         // 1-D length; 0 for 2-D
    int Hh, Ww;                    // 2-D grid; 0 for 1-D
    int n_bands;
    float inv_div;                 // 1 / decay_div
    float* h;                      // [rows][positions]
};

constexpr int kFgTile = 64;        // positions per head CTA
constexpr int kFgRowTile = 128;    // head rows per CTA
constexpr int kFgThreads = 256;
constexpr int kFgLayerPos = 16;    // positions per layers CTA (16 threads each)
constexpr int kFgAS = kFgTile + 1; // activation row stride
constexpr int kFgOS = kFfnWidth + 1;
// weight row strides: odd, so the units the threads of one position read
// at once sit on different banks
constexpr int kFgW1S = kFfnMaxIn + 1;
constexpr int kFgWS = kFfnWidth + 1;
constexpr int kFgWRegion = kFfnWidth * kFgW1S + 2 * kFfnWidth * kFgWS;
// layers kernel shared memory (floats): weights + two activation buffers
constexpr size_t kFgLayerSmemBytes = sizeof(float) * (kFgWRegion + 2 * kFfnWidth * (kFgLayerPos + 1));
// head kernel shared memory (floats): the Wout tile transposed [64][132]
// and the a3 tile [64][68]; rows 16-byte aligned for 128-bit loads
constexpr int kFgWTS = kFgRowTile + 4;
constexpr int kFgA4S = kFgTile + 4;
constexpr size_t kFgHeadSmemBytes = sizeof(float) * (kFfnWidth * kFgWTS + kFfnWidth * kFgA4S);
// tail kernel: 16 positions x the 64 stash rows per CTA
constexpr int kFgTailPos = 16;
constexpr size_t kFgTailSmemBytes = sizeof(float) * (kFfnWidth * kFgOS + kFfnWidth * (kFgTailPos + 1));
// single-launch path (few rows): weights + Wout tile + two activation tiles
constexpr size_t kFgFusedSmemBytes = sizeof(float) * (kFgWRegion + 2 * kFfnWidth * kFgAS);
static_assert(kFgRowTile * kFgOS <= kFgWRegion, "Wout tile fits the weight region");

// Positional features of position `pos` in the canonical slots (1-D:
// [t, (sin, cos) band 1..16]; 2-D: [ty, tx, (sin, cos) y-band 1..16,
// (sin, cos) x-band 1..16]).
template <bool TWO_D>
__device__ __forceinline__ void features(const FilterGenArgs& a, long pos, float* phi)
{
#pragma unroll
    for (int c = 0; c < kFfnMaxIn; ++c) phi[c] = 0.0f;
    if constexpr (!TWO_D) {
        const int i = (int)pos;
        phi[0] = (float)i / (float)a.L;
#pragma unroll
        for (int k = 1; k <= 16; ++k) {
            if (k > a.n_bands) break;
            // angle 2 pi k i / L reduced exactly: 2 pi ((k i) mod L) / L
            const int qk = (int)(((long)k * i) % a.L);
            float sn, cs;
            sincospif(2.0f * (float)qk / (float)a.L, &sn, &cs);
            phi[2 * k - 1] = sn;
            phi[2 * k] = cs;
        }
    } else {
        const int iy = (int)(pos / a.Ww), ix = (int)(pos % a.Ww);
        phi[0] = (float)iy / (float)a.Hh;
        phi[1] = (float)ix / (float)a.Ww;
#pragma unroll
        for (int k = 1; k <= 16; ++k) {
            if (k > a.n_bands) break;
            float sn, cs;
            const int qy = (int)(((long)k * iy) % a.Hh);
            sincospif(2.0f * (float)qy / (float)a.Hh, &sn, &cs);
            phi[2 * k] = sn;
            phi[2 * k + 1] = cs;
            const int qx = (int)(((long)k * ix) % a.Ww);
            sincospif(2.0f * (float)qx / (float)a.Ww, &sn, &cs);
            phi[2 + 2 * 16 + 2 * (k - 1)] = sn;
            phi[2 + 2 * 16 + 2 * (k - 1) + 1] = cs;
        }
    }
}

// Stage W1 (canonical feature slots), W2, W3 into shared memory, zero
// padded to 64 units (sin(0) = 0: padded units contribute nothing).
template <bool TWO_D>
__device__ __forceinline__ void stage_weights(const FilterGenArgs& a, float* sW1, float* sW2, float* sW3)
{
    const int tid = threadIdx.x;
    for (int e = tid; e < kFfnWidth * kFfnMaxIn; e += blockDim.x) {
        const int r = e / kFfnMaxIn, c = e % kFfnMaxIn;
        int src = -1;
        if constexpr (!TWO_D) {
            src = c < a.n_in ? c : -1;
        } else {
            constexpr int XB = 2 + 2 * 16;   // slot of the first x-band feature
            if (c < 2 + 2 * a.n_bands) src = c;
            else if (c >= XB && c < XB + 2 * a.n_bands) src = 2 + 2 * a.n_bands + (c - XB);
        }
        sW1[r * kFgW1S + c] = (r < a.width && src >= 0) ? __ldg(a.W1 + r * a.n_in + src) : 0.0f;
    }
    for (int e = tid; e < kFfnWidth * kFfnWidth; e += blockDim.x) {
        const int r = e / kFfnWidth, c = e % kFfnWidth;
        const bool in = r < a.width && c < a.width;
        sW2[r * kFgWS + c] = in ? __ldg(a.W2 + r * a.width + c) : 0.0f;
        sW3[r * kFgWS + c] = in ? __ldg(a.W3 + r * a.width + c) : 0.0f;
    }
}

// The three sine layers for position p of a tile: UPT = 64 / TPP output
// units per thread, TPP threads per position (thread q of the position owns
// units TPP * jj + q).  a1 and a3 end up in sA[j * AS + p], a2 in sB.
template <bool TWO_D, int TPP, int AS>
__device__ __forceinline__ void sine_layers(const FilterGenArgs& a, long pos, int p, int q,
                                            const float* sW1, const float* sW2, const float* sW3,
                                            float* sA, float* sB)
{
    constexpr int UPT = kFfnWidth / TPP;
    constexpr int NIN = TWO_D ? kFfnMaxIn : 33;        // 1-D features use slots < 33
    {
        float phi[kFfnMaxIn];
        features<TWO_D>(a, pos, phi);
        __syncthreads();                                   // weights staged by all threads
        float acc[UPT];
#pragma unroll
        for (int jj = 0; jj < UPT; ++jj) acc[jj] = 0.0f;
#pragma unroll
        for (int c = 0; c < NIN; ++c)
#pragma unroll
            for (int jj = 0; jj < UPT; ++jj)
                acc[jj] = fmaf(sW1[(TPP * jj + q) * kFgW1S + c], phi[c], acc[jj]);
#pragma unroll
        for (int jj = 0; jj < UPT; ++jj) sA[(TPP * jj + q) * AS + p] = sinf(acc[jj]);
    }
    __syncthreads();
#pragma unroll 1
    for (int layer = 0; layer < 2; ++layer) {
        const float* Wl = layer == 0 ? sW2 : sW3;
        const float* in = layer == 0 ? sA : sB;
        float* out = layer == 0 ? sB : sA;
        float acc[UPT];
#pragma unroll
        for (int jj = 0; jj < UPT; ++jj) acc[jj] = 0.0f;
#pragma unroll 8
        for (int c = 0; c < kFfnWidth; ++c) {
            const float x = in[c * AS + p];
#pragma unroll
            for (int jj = 0; jj < UPT; ++jj) acc[jj] = fmaf(Wl[(TPP * jj + q) * kFgWS + c], x, acc[jj]);
        }
#pragma unroll
        for (int jj = 0; jj < UPT; ++jj) out[(TPP * jj + q) * AS + p] = sinf(acc[jj]);
        __syncthreads();
    }
}

// Head for rows r0 .. r0+127 (< r_end) and positions p0 .. p0+63 from the
// a3 tile in sA [64][kFgAS] and the Wout tile staged into sOut.
template <bool TWO_D>
__device__ __forceinline__ void head_tile(const FilterGenArgs& a, long npos, long p0, int r0, int r_end,
                                          float* sOut, const float* sA)
{
    const int tid = threadIdx.x;
    for (int e = tid; e < kFgRowTile * kFfnWidth; e += kFgThreads) {
        const int r = e / kFfnWidth, j = e % kFfnWidth;
        sOut[r * kFgOS + j] = (r0 + r < r_end && j < a.width)
                                  ? __ldg(a.Wout + (long)(r0 + r) * a.width + j) : 0.0f;
    }
    __syncthreads();
    // thread (ty, tx) of a 16 x 16 grid: rows ty + 16 i (i < 8), positions tx + 16 k (k < 4)
    const int tx = tid % 16, ty = tid / 16;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[i][k] = 0.0f;
#pragma unroll 4
    for (int j = 0; j < kFfnWidth; ++j) {
        float w[8], x[4];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = sOut[(ty + 16 * i) * kFgOS + j];
#pragma unroll
        for (int k = 0; k < 4; ++k) x[k] = sA[j * kFgAS + tx + 16 * k];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[i][k] = fmaf(w[i], x[k], acc[i][k]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = r0 + ty + 16 * i;
        if (r >= r_end) continue;
        const float al = __ldg(a.alpha + r % a.D);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const long pos = p0 + tx + 16 * k;
            if (pos >= npos) continue;
            float dist;   // the window's argument: i (1-D) or iy + ix (2-D)
            if constexpr (!TWO_D) dist = (float)pos;
            else dist = (float)(pos / a.Ww) + (float)(pos % a.Ww);
            a.h[(long)r * npos + pos] = acc[i][k] * expf(-al * dist * a.inv_div);
        }
    }
}

// Layers kernel: a3 of 16 positions into the stash rows (the last 64 rows
// of h), a3[j][pos] at h[(rows - 64 + j) * npos + pos].
template <bool TWO_D>
__global__ void __launch_bounds__(kFgThreads) filter_layers_kernel(FilterGenArgs a)
{
    extern __shared__ __align__(16) float fg_smem[];
    constexpr int AS = kFgLayerPos + 1;
    float* sW1 = fg_smem;
    float* sW2 = sW1 + kFfnWidth * kFgW1S;
    float* sW3 = sW2 + kFfnWidth * kFgWS;
    float* sA = fg_smem + kFgWRegion;
    float* sB = sA + kFfnWidth * AS;
    const long npos = TWO_D ? (long)a.Hh * a.Ww : (long)a.L;
    const long p0 = (long)blockIdx.x * kFgLayerPos;
    const int p = threadIdx.x / 16, q = threadIdx.x % 16;
    stage_weights<TWO_D>(a, sW1, sW2, sW3);
    sine_layers<TWO_D, 16, AS>(a, min(p0 + p, npos - 1), p, q, sW1, sW2, sW3, sA, sB);
    // stash a3 (coalesced along the position)
    float* stash = a.h + (long)(a.rows - kFfnWidth) * npos;
    for (int e = threadIdx.x; e < kFfnWidth * kFgLayerPos; e += kFgThreads) {
        const int j = e / kFgLayerPos, pp = e % kFgLayerPos;
        if (p0 + pp < npos) stash[(long)j * npos + p0 + pp] = sA[j * AS + pp];
    }
}

// Head kernel: rows 0 .. rows-65 as 128-row x 64-position tiles (grid.y
// over row tiles).  Thread (ty, tx) computes rows 8 ty + i (i < 8) and
// positions 4 tx + k (k < 4): per unit j one 128-bit load of 4 a3 values and
// two of 8 Wout values for 32 multiply-adds.
template <bool TWO_D>
__global__ void __launch_bounds__(kFgThreads) filter_head_kernel(FilterGenArgs a)
{
    extern __shared__ __align__(16) float fg_smem[];
    float* sWT = fg_smem;                                   // [64][132]: Wout tile, transposed
    float* sA = fg_smem + kFfnWidth * kFgWTS;               // [64][68]:  a3 tile
    const long npos = TWO_D ? (long)a.Hh * a.Ww : (long)a.L;
    const long p0 = (long)blockIdx.x * kFgTile;
    const int r0 = blockIdx.y * kFgRowTile;
    const int stash_row = a.rows - kFfnWidth;
    const float* stash = a.h + (long)stash_row * npos;
    const int tid = threadIdx.x;
    for (int e = tid; e < kFfnWidth * kFgTile; e += kFgThreads) {
        const int j = e / kFgTile, pp = e % kFgTile;
        sA[j * kFgA4S + pp] = p0 + pp < npos ? stash[(long)j * npos + p0 + pp] : 0.0f;
    }
    for (int e = tid; e < kFgRowTile * kFfnWidth; e += kFgThreads) {
        const int r = e / kFfnWidth, j = e % kFfnWidth;
        sWT[j * kFgWTS + r] = (r0 + r < stash_row && j < a.width)
                                  ? __ldg(a.Wout + (long)(r0 + r) * a.width + j) : 0.0f;
    }
    __syncthreads();
    const int tx = tid % 16, ty = tid / 16;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[i][k] = 0.0f;
#pragma unroll 4
    for (int j = 0; j < kFfnWidth; ++j) {
        const float4 x4 = *reinterpret_cast<const float4*>(sA + j * kFgA4S + 4 * tx);
        const float4 w0 = *reinterpret_cast<const float4*>(sWT + j * kFgWTS + 8 * ty);
        const float4 w1 = *reinterpret_cast<const float4*>(sWT + j * kFgWTS + 8 * ty + 4);
        const float w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        const float x[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[i][k] = fmaf(w[i], x[k], acc[i][k]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = r0 + 8 * ty + i;
        if (r >= stash_row) continue;
        const float al = __ldg(a.alpha + r % a.D);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const long pos = p0 + 4 * tx + k;
            if (pos >= npos) continue;
            float dist;   // the window's argument: i (1-D) or iy + ix (2-D)
            if constexpr (!TWO_D) dist = (float)pos;
            else dist = (float)(pos / a.Ww) + (float)(pos % a.Ww);
            a.h[(long)r * npos + pos] = acc[i][k] * expf(-al * dist * a.inv_div);
        }
    }
}

// Tail kernel: the 64 stash rows for 16 positions per CTA; each CTA reads
// its own 64 x 16 tile of a3 before overwriting exactly that tile.
template <bool TWO_D>
__global__ void __launch_bounds__(kFgThreads) filter_tail_kernel(FilterGenArgs a)
{
    extern __shared__ __align__(16) float fg_smem[];
    constexpr int AS = kFgTailPos + 1;
    float* sW = fg_smem;                                    // [64][65]: Wout stash rows
    float* sA = fg_smem + kFfnWidth * kFgOS;                // [64][17]: a3 tile
    const long npos = TWO_D ? (long)a.Hh * a.Ww : (long)a.L;
    const long p0 = (long)blockIdx.x * kFgTailPos;
    const int stash_row = a.rows - kFfnWidth;
    float* stash = a.h + (long)stash_row * npos;
    const int tid = threadIdx.x;
    for (int e = tid; e < kFfnWidth * kFgTailPos; e += kFgThreads) {
        const int j = e / kFgTailPos, pp = e % kFgTailPos;
        sA[j * AS + pp] = p0 + pp < npos ? stash[(long)j * npos + p0 + pp] : 0.0f;
    }
    for (int e = tid; e < kFfnWidth * kFfnWidth; e += kFgThreads) {
        const int r = e / kFfnWidth, j = e % kFfnWidth;
        sW[r * kFgOS + j] = j < a.width ? __ldg(a.Wout + (long)(stash_row + r) * a.width + j) : 0.0f;
    }
    __syncthreads();
    // thread (ty, tx): rows ty + 16 i (i < 4), position tx
    const int tx = tid % 16, ty = tid / 16;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 8
    for (int j = 0; j < kFfnWidth; ++j) {
        const float x = sA[j * AS + tx];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] = fmaf(sW[(ty + 16 * i) * kFgOS + j], x, acc[i]);
    }
    const long pos = p0 + tx;
    if (pos >= npos) return;
    float dist;
    if constexpr (!TWO_D) dist = (float)pos;
    else dist = (float)(pos / a.Ww) + (float)(pos % a.Ww);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = stash_row + ty + 16 * i;
        const float al = __ldg(a.alpha + r % a.D);
        stash[(long)(ty + 16 * i) * npos + pos] = acc[i] * expf(-al * dist * a.inv_div);
    }
}

// Single launch for few rows (< 64 + 1): every CTA evaluates the layers of
// its 64 positions, then the head for all rows.
template <bool TWO_D>
__global__ void __launch_bounds__(kFgThreads) filter_gen_kernel(FilterGenArgs a)
{
    extern __shared__ __align__(16) float fg_smem[];
    float* sW1 = fg_smem;
    float* sW2 = sW1 + kFfnWidth * kFgW1S;
    float* sW3 = sW2 + kFfnWidth * kFgWS;
    float* sOut = fg_smem;                                   // after the layers
    float* sA = fg_smem + kFgWRegion;
    float* sB = sA + kFfnWidth * kFgAS;
    const long npos = TWO_D ? (long)a.Hh * a.Ww : (long)a.L;
    const long p0 = (long)blockIdx.x * kFgTile;
    const int p = threadIdx.x / 4, q = threadIdx.x % 4;
    stage_weights<TWO_D>(a, sW1, sW2, sW3);
    sine_layers<TWO_D, 4, kFgAS>(a, min(p0 + p, npos - 1), p, q, sW1, sW2, sW3, sA, sB);
    head_tile<TWO_D>(a, npos, p0, 0, a.rows, sOut, sA);
}

}  // namespace hyena
