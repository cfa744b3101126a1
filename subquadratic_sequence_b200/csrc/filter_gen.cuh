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
// Every stage is a small dense product evaluated as a register-tiled SIMT
// GEMM out of shared memory (each thread owns a 4 x 4 or 8 x 4 block of
// outputs: one 128-bit load of weights and one of activations per 16 or 32
// multiply-adds).  Three launches, no recomputation:
//  layers: a persistent kernel (weights staged once per CTA) evaluates the
//          three sine layers for tiles of positions and stashes
//          a3 [64][positions] in the LAST 64 rows of h (they are outputs
//          too, written last);
//  head:   h[r][p] = (sum_j Wout[r][j] a3[j][p]) * window for the rows
//          before the stash, as 128-row x 64-position tiles;
//  tail:   the head for the 64 stash rows, 64 positions per CTA: each CTA
//          loads its own tile of a3 into shared memory before overwriting
//          exactly that tile.
// With at most 64 rows the layers are evaluated inside the head kernel
// instead (one launch).  The sine is the hardware approximation __sinf:
// the arguments are sums of 17 to 66 products of N(0, 1/fan_in) weights
// with values in [-1, 1], so they stay within a few units of zero, where
// its absolute error is below 1e-6.
#pragma once

#include "hyena_common.cuh"

namespace hyena {

constexpr int kFfnWidth = 64;      // widths above this are rejected
constexpr int kFfnMaxIn = 66;      // 2 + 4 * 16 bands

struct FilterGenArgs {
    const float *W1, *W2, *W3, *Wout, *alpha;
    int n_in, width, rows;         // rows = N * D
    int D;                         // channels (alpha index = row % D)
    int L;                         // 1-D length; 0 for 2-D and 3-D
    int Hh, Ww;                    // 2-D grid (the planes of a 3-D volume); 0 for 1-D
    int Zz;                        // 3-D volume depth; 0 for 1-D and 2-D (3-D runs the 2-D kernels)
    int n_bands;
    float inv_div;                 // 1 / decay_div
    float* h;                      // [rows][positions] (per sample with FiLM)
    int vec;                       // positions % 4 == 0 and h 16-byte aligned: 128-bit h access
    // input-dependent filters (1-D): sample b = blockIdx.z modulates the
    // sine layers, a_l = sin(omega_l (gamma_bl (W_l a_(l-1)) + beta_bl));
    // NULL omega / gamma / beta mean 1 / 1 / 0
    const float *omega;            // [3][width]
    const float *gamma, *beta;     // [B][3][width]
    int film;                      // 1: modulate (any of the three given)
    int gaussian;                  // 1: window exp(-t^2 / (2 sigma^2)), sigma in alpha[]
    float inv_L, inv_H, inv_W;     // 1/L (1-D), 1/H and 1/W (2-D): t = i/L, ty = iy/H, tx = ix/W
    float inv_Z;                   // 1/Z (3-D): tz = iz/Z
    long sample_stride;            // floats of h per sample (rows * positions)
};

// The window of a row is exp(c u): the exponential decay has u = i (1-D)
// or iy + ix (2-D) and c = -alpha / div; the Gaussian has u = t^2 (1-D) or
// ty^2 + tx^2 (2-D) and c = -1 / (2 sigma^2).  par is alpha or sigma.
__device__ __forceinline__ float window_coeff(const FilterGenArgs& a, float par)
{
    return a.gaussian ? -0.5f / (par * par) : -par * a.inv_div;
}

// Offsets the per-sample pointers by the sample of this CTA (blockIdx.z).
__device__ __forceinline__ void select_sample(FilterGenArgs& a)
{
    const int b = blockIdx.z;
    a.h += (long)b * a.sample_stride;
    if (a.gamma) a.gamma += (long)b * 3 * a.width;
    if (a.beta) a.beta += (long)b * 3 * a.width;
}

// Positions of one filter: L (1-D), H W (2-D) or Z H W (3-D).
template <bool TWO_D>
__device__ __forceinline__ long fg_positions(const FilterGenArgs& a)
{
    if constexpr (!TWO_D) return (long)a.L;
    else return (long)(a.Zz ? a.Zz : 1) * a.Hh * a.Ww;
}

// 3-D feature slots (n_bands <= 10): [tz, ty, tx], then per axis a (z, y,
// x) and band b = 1..10 the pair (sin, cos) at 3 + 20 a + 2 (b - 1).
constexpr int kFg3dBands = 10;

constexpr int kFgThreads = 256;     // a 16 x 16 thread grid
constexpr int kFgTile = 64;         // positions per head / tail / layers tile
constexpr int kFgRowTile = 128;     // head rows per CTA
constexpr int kFgSmallTile = 16;    // positions per layers tile for short filters
// shared-memory row strides (floats): multiples of 4, so every row starts
// 16-byte aligned for 128-bit loads
constexpr int kFgUS = kFfnWidth + 4;     // [input][unit] weight rows, [unit][pos] tiles of 64
constexpr int kFgRS = kFgRowTile + 4;    // [unit][row] Wout tile of the head
// transposed W1 (canonical feature slots), W2, W3: [input][unit]
constexpr int kFgWRegion = (kFfnMaxIn + 2 * kFfnWidth) * kFgUS;
// FiLM parameters of the three layers: [layer][omega, gamma, beta][unit]
constexpr int kFgFilm = 3 * 3 * kFfnWidth;

template <int PT>
struct LayerTile {
    static constexpr int AS = PT + 4;                    // activation row stride
    static constexpr int PPT = PT / 16;                  // positions per thread
    // weights + features/a2 [66][AS] + a1/a3 [64][AS] + FiLM [3][3][64]
    static constexpr size_t SMEM = sizeof(float) * (kFgWRegion + (kFfnMaxIn + kFfnWidth) * AS + kFgFilm);
};
template <int NG>
constexpr size_t fg_head_smem_bytes() { return sizeof(float) * (kFfnWidth * kFgRS + kFfnWidth * (64 * NG + 4)); }
constexpr size_t kFgTailSmemBytes = sizeof(float) * 2 * kFfnWidth * kFgUS;
constexpr size_t kFgTail16SmemBytes = sizeof(float) * kFfnWidth * (kFgUS + kFgSmallTile + 4);
// single launch (rows <= 64): layers tile of 64 positions, then the head;
// the Wout rows reuse the weight region
constexpr size_t kFgFusedSmemBytes = LayerTile<kFgTile>::SMEM;
static_assert(kFfnWidth * kFgUS <= kFgWRegion, "Wout rows fit the weight region");

// Positional features of the tile's positions p0 .. p0+PT-1 into sX[slot][p]
// (1-D slots: [t, (sin, cos) band 1..16]; 2-D: [ty, tx, (sin, cos) y-band
// 1..16, (sin, cos) x-band 1..16]); bands above n_bands and positions past
// the end are zero.
template <bool TWO_D, int PT>
__device__ __forceinline__ void features_tile(const FilterGenArgs& a, long npos, long p0, float* sX)
{
    constexpr int AS = LayerTile<PT>::AS;
    const int tid = threadIdx.x;
    if constexpr (!TWO_D) {
        for (int e = tid; e < 17 * PT; e += kFgThreads) {
            const int k = e / PT, p = e % PT;
            const long pos = p0 + p;
            const int i = (int)pos;
            if (k == 0) {
                sX[p] = pos < npos ? (float)i / (float)a.L : 0.0f;
            } else {
                float sn = 0.0f, cs = 0.0f;
                if (k <= a.n_bands && pos < npos) {
                    // angle 2 pi k i / L reduced exactly: 2 pi ((k i) mod L) / L
                    const int qk = (int)(((long)k * i) % a.L);
                    sincospif(2.0f * (float)qk / (float)a.L, &sn, &cs);
                }
                sX[(2 * k - 1) * AS + p] = sn;
                sX[(2 * k) * AS + p] = cs;
            }
        }
    } else if (a.Zz) {
        for (int e = tid; e < (1 + 3 * kFg3dBands) * PT; e += kFgThreads) {
            const int k = e / PT, p = e % PT;
            const long pos = p0 + p;
            const int ip = (int)pos, iz = ip / (a.Hh * a.Ww), iyx = ip - iz * (a.Hh * a.Ww);
            const int iy = iyx / a.Ww, ix = iyx - iy * a.Ww;
            if (k == 0) {
                sX[p] = pos < npos ? (float)iz / (float)a.Zz : 0.0f;
                sX[AS + p] = pos < npos ? (float)iy / (float)a.Hh : 0.0f;
                sX[2 * AS + p] = pos < npos ? (float)ix / (float)a.Ww : 0.0f;
            } else {
                const int axis = (k - 1) / kFg3dBands, band = (k - 1) % kFg3dBands + 1;
                float sn = 0.0f, cs = 0.0f;
                if (band <= a.n_bands && pos < npos) {
                    const int n = axis == 0 ? a.Zz : (axis == 1 ? a.Hh : a.Ww);
                    const int c = axis == 0 ? iz : (axis == 1 ? iy : ix);
                    const int qk = (int)(((long)band * c) % n);
                    sincospif(2.0f * (float)qk / (float)n, &sn, &cs);
                }
                const int slot = 3 + 2 * kFg3dBands * axis + 2 * (band - 1);
                sX[slot * AS + p] = sn;
                sX[(slot + 1) * AS + p] = cs;
            }
        }
        // slots 63 .. kFfnMaxIn - 1 are never written: their W1 rows are zero
        for (int e = tid; e < (kFfnMaxIn - 3 - 6 * kFg3dBands) * PT; e += kFgThreads)
            sX[(3 + 6 * kFg3dBands + e / PT) * AS + e % PT] = 0.0f;
    } else {
        constexpr int XB = 2 + 2 * 16;                  // slot of the first x-band feature
        for (int e = tid; e < 33 * PT; e += kFgThreads) {
            const int k = e / PT, p = e % PT;
            const long pos = p0 + p;
            const int ip = (int)pos, iy = ip / a.Ww, ix = ip - iy * a.Ww;   // positions < 2^30
            if (k == 0) {
                sX[p] = pos < npos ? (float)iy / (float)a.Hh : 0.0f;
                sX[AS + p] = pos < npos ? (float)ix / (float)a.Ww : 0.0f;
            } else {
                const int band = (k - 1) % 16 + 1;
                const bool xaxis = k > 16;
                float sn = 0.0f, cs = 0.0f;
                if (band <= a.n_bands && pos < npos) {
                    const int n = xaxis ? a.Ww : a.Hh, c = xaxis ? ix : iy;
                    const int qk = (int)(((long)band * c) % n);
                    sincospif(2.0f * (float)qk / (float)n, &sn, &cs);
                }
                const int slot = xaxis ? XB + 2 * (band - 1) : 2 * band;
                sX[slot * AS + p] = sn;
                sX[(slot + 1) * AS + p] = cs;
            }
        }
    }
}

// Stage W1 (canonical feature slots), W2, W3 transposed into shared memory
// as [input][unit], zero padded to 64 units (sin(0) = 0: padded units
// contribute nothing).  All loads of a matrix are issued before its stores.
template <bool TWO_D>
__device__ __forceinline__ void stage_weights(const FilterGenArgs& a, float* sW)
{
    constexpr int NIN = TWO_D ? kFfnMaxIn : 33;
    const int tid = threadIdx.x;
    float* sW1 = sW;
    float* sW2 = sW + kFfnMaxIn * kFgUS;
    float* sW3 = sW2 + kFfnWidth * kFgUS;
    {
        constexpr int PER = (kFfnWidth * NIN + kFgThreads - 1) / kFgThreads;
        float v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = tid + i * kFgThreads;
            const int u = e / NIN, c = e % NIN;
            int src = -1;
            if constexpr (!TWO_D) {
                src = c < a.n_in ? c : -1;
            } else if (a.Zz) {
                // canonical 3-D slot -> W1 column [tz, ty, tx, z bands, y bands, x bands]
                if (c < 3) {
                    src = c;
                } else if (c < 3 + 6 * kFg3dBands) {
                    const int axis = (c - 3) / (2 * kFg3dBands), rem = (c - 3) % (2 * kFg3dBands);
                    if (rem < 2 * a.n_bands) src = 3 + 2 * a.n_bands * axis + rem;
                }
            } else {
                constexpr int XB = 2 + 2 * 16;
                if (c < 2 + 2 * a.n_bands) src = c;
                else if (c >= XB && c < XB + 2 * a.n_bands) src = 2 + 2 * a.n_bands + (c - XB);
            }
            v[i] = (e < kFfnWidth * NIN && u < a.width && src >= 0) ? __ldg(a.W1 + u * a.n_in + src) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = tid + i * kFgThreads;
            if (e < kFfnWidth * NIN) sW1[(e % NIN) * kFgUS + e / NIN] = v[i];
        }
    }
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const float* W = m == 0 ? a.W2 : a.W3;
        float* dst = m == 0 ? sW2 : sW3;
        constexpr int PER = kFfnWidth * kFfnWidth / kFgThreads;
        float v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = tid + i * kFgThreads;
            const int u = e / kFfnWidth, c = e % kFfnWidth;
            v[i] = (u < a.width && c < a.width) ? __ldg(W + u * a.width + c) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = tid + i * kFgThreads;
            dst[(e % kFfnWidth) * kFgUS + e / kFfnWidth] = v[i];
        }
    }
}

// out[u][p] = sin(sum_c W[u][c] in[c][p]) for 64 units and the PT positions
// of a tile; thread (ty, tx) owns units 4 ty .. 4 ty + 3 and positions
// PPT tx .. PPT tx + PPT - 1.  WT is [input][unit] (stride kFgUS).
template <int PT, int K>
__device__ __forceinline__ void sine_layer(const float* WT, const float* in, float* out, const float* film)
{
    constexpr int AS = LayerTile<PT>::AS, PPT = LayerTile<PT>::PPT;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][PPT];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int k = 0; k < PPT; ++k) acc[i][k] = 0.0f;
#pragma unroll 11
    for (int c = 0; c < K; ++c) {
        const float4 w = *reinterpret_cast<const float4*>(WT + c * kFgUS + 4 * ty);
        float x[PPT];
        if constexpr (PPT == 4) {
            const float4 x4 = *reinterpret_cast<const float4*>(in + c * AS + 4 * tx);
            x[0] = x4.x; x[1] = x4.y; x[2] = x4.z; x[3] = x4.w;
        } else {
            x[0] = in[c * AS + tx];
        }
        const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k = 0; k < PPT; ++k) acc[i][k] = fmaf(wv[i], x[k], acc[i][k]);
    }
    if (film) {
        // feature-wise modulation of this layer: omega (gamma acc + beta)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int u = 4 * ty + i;
            const float om = film[u], g = film[kFfnWidth + u], be = film[2 * kFfnWidth + u];
#pragma unroll
            for (int k = 0; k < PPT; ++k) acc[i][k] = om * fmaf(g, acc[i][k], be);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if constexpr (PPT == 4) {
            *reinterpret_cast<float4*>(out + (4 * ty + i) * AS + 4 * tx) =
                make_float4(__sinf(acc[i][0]), __sinf(acc[i][1]), __sinf(acc[i][2]), __sinf(acc[i][3]));
        } else {
            out[(4 * ty + i) * AS + tx] = __sinf(acc[i][0]);
        }
    }
}

// Stage the FiLM parameters of this CTA's sample into sF [3][3][64]
// (omega, gamma, beta per layer; defaults 1, 1, 0).
__device__ __forceinline__ void stage_film(const FilterGenArgs& a, float* sF)
{
    for (int e = threadIdx.x; e < kFgFilm; e += blockDim.x) {
        const int l = e / (3 * kFfnWidth), kind = (e / kFfnWidth) % 3, u = e % kFfnWidth;
        float v = kind == 2 ? 0.0f : 1.0f;
        if (u < a.width) {
            const float* src = kind == 0 ? a.omega : kind == 1 ? a.gamma : a.beta;
            if (src) v = __ldg(src + l * a.width + u);
        }
        sF[e] = v;
    }
}

// The three sine layers of one tile: features into sX, a1 into sY, a2 into
// sX, a3 into sY.  Ends with a barrier (a3 visible to the whole CTA).
template <bool TWO_D, int PT>
__device__ __forceinline__ void layers_tile(const FilterGenArgs& a, long npos, long p0, const float* sW,
                                            float* sX, float* sY, const float* sF)
{
    constexpr int NIN = TWO_D ? kFfnMaxIn : 33;
    const float* f = a.film ? sF : nullptr;
    features_tile<TWO_D, PT>(a, npos, p0, sX);
    __syncthreads();
    sine_layer<PT, NIN>(sW, sX, sY, f);
    __syncthreads();
    sine_layer<PT, kFfnWidth>(sW + kFfnMaxIn * kFgUS, sY, sX, f ? f + 3 * kFfnWidth : nullptr);
    __syncthreads();
    sine_layer<PT, kFfnWidth>(sW + (kFfnMaxIn + kFfnWidth) * kFgUS, sX, sY, f ? f + 6 * kFfnWidth : nullptr);
    __syncthreads();
}

// The window's argument u at position pos (positions are below 2^30).
template <bool TWO_D>
__device__ __forceinline__ float window_u(const FilterGenArgs& a, long pos)
{
    if constexpr (!TWO_D) {
        if (a.gaussian) {
            const float t = (float)pos * a.inv_L;
            return t * t;
        }
        return (float)pos;
    } else {
        int ip = (int)pos, iz = 0;
        if (a.Zz) {
            iz = ip / (a.Hh * a.Ww);
            ip -= iz * (a.Hh * a.Ww);
        }
        const int iy = ip / a.Ww, ix = ip - iy * a.Ww;
        if (a.gaussian) {
            const float tz = (float)iz * a.inv_Z, ty = (float)iy * a.inv_H, tx = (float)ix * a.inv_W;
            return tz * tz + ty * ty + tx * tx;
        }
        return (float)(iz + iy + ix);
    }
}

// Load a [64][64 NG] tile of a3 (positions p0 .. p0 + 64 NG - 1 of the
// stash rows) into sA [64][64 NG + 4]; positions past the end read as zero.
template <int NG>
__device__ __forceinline__ void load_a3_tile(const FilterGenArgs& a, long npos, long p0, const float* stash,
                                             float* sA)
{
    constexpr int PT = 64 * NG, AS = PT + 4;
    const int tid = threadIdx.x;
    if (a.vec) {
        constexpr int PER = kFfnWidth * PT / 4 / kFgThreads;
        float4 v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = tid + i * kFgThreads, j = e / (PT / 4), q = e % (PT / 4);
            const long pos = p0 + 4 * q;
            v[i] = pos < npos ? *reinterpret_cast<const float4*>(stash + (long)j * npos + pos)
                              : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = tid + i * kFgThreads, j = e / (PT / 4), q = e % (PT / 4);
            *reinterpret_cast<float4*>(sA + j * AS + 4 * q) = v[i];
        }
    } else {
        constexpr int PER = kFfnWidth * PT / kFgThreads;
        float v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = tid + i * kFgThreads, j = e / PT, pp = e % PT;
            v[i] = p0 + pp < npos ? stash[(long)j * npos + p0 + pp] : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = tid + i * kFgThreads;
            sA[(e / PT) * AS + e % PT] = v[i];
        }
    }
}

// Stage rows r0 .. r0 + NR - 1 (< r_end) of Wout transposed into
// sWT [64][RS] (zero past r_end and past the width).
template <int NR, int RS>
__device__ __forceinline__ void load_wout_tile(const FilterGenArgs& a, int r0, int r_end, float* sWT)
{
    constexpr int PER = NR * kFfnWidth / kFgThreads;
    const int tid = threadIdx.x;
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = tid + i * kFgThreads, r = e / kFfnWidth, j = e % kFfnWidth;
        v[i] = (r0 + r < r_end && j < a.width) ? __ldg(a.Wout + (long)(r0 + r) * a.width + j) : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = tid + i * kFgThreads;
        sWT[(e % kFfnWidth) * RS + e / kFfnWidth] = v[i];
    }
}

// h[r][p] = (sum_j Wout[r][j] a3[j][p]) * window for rows r0 + RT ty + i
// (i < RT, r < r_end) and positions p0 + 64 g + 4 tx + k (g < NG, k < 4)
// from sWT [64][RS] and sA [64][64 NG + 4] (each 128-bit load of a3 is then
// contiguous across the 16 tx); alpha of the thread's rows is passed in.
template <bool TWO_D, int RT, int RS, int NG>
__device__ __forceinline__ void head_block(const FilterGenArgs& a, long npos, long p0, int r0, int r_end,
                                           const float* sWT, const float* sA, const float* al)
{
    constexpr int AS = 64 * NG + 4;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[RT][4 * NG];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int k = 0; k < 4 * NG; ++k) acc[i][k] = 0.0f;
#pragma unroll 8
    for (int j = 0; j < kFfnWidth; ++j) {
        float x[4 * NG], w[RT];
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const float4 x4 = *reinterpret_cast<const float4*>(sA + j * AS + 64 * g + 4 * tx);
            x[4 * g] = x4.x; x[4 * g + 1] = x4.y; x[4 * g + 2] = x4.z; x[4 * g + 3] = x4.w;
        }
#pragma unroll
        for (int i = 0; i < RT; i += 4) {
            const float4 w4 = *reinterpret_cast<const float4*>(sWT + j * RS + RT * ty + i);
            w[i] = w4.x; w[i + 1] = w4.y; w[i + 2] = w4.z; w[i + 3] = w4.w;
        }
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
            for (int k = 0; k < 4 * NG; ++k) acc[i][k] = fmaf(w[i], x[k], acc[i][k]);
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        const long pos0 = p0 + 64 * g + 4 * tx;
            float dist[4];   // window arguments of the group's 4 positions
#pragma unroll
        for (int k = 0; k < 4; ++k) dist[k] = window_u<TWO_D>(a, pos0 + k);
#pragma unroll
        for (int i = 0; i < RT; ++i) {
            const int r = r0 + RT * ty + i;
            if (r >= r_end) continue;
            float* hr = a.h + (long)r * npos;
            const float* v = acc[i] + 4 * g;
            float wv[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) wv[k] = v[k] * expf(al[i] * dist[k]);
            if (a.vec) {
                if (pos0 < npos) *reinterpret_cast<float4*>(hr + pos0) = make_float4(wv[0], wv[1], wv[2], wv[3]);
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (pos0 + k < npos) hr[pos0 + k] = wv[k];
            }
        }
    }
}

// Window coefficients of rows r0 + RT ty + i (loaded before the products
// so the loads overlap them).
template <int RT>
__device__ __forceinline__ void load_alpha(const FilterGenArgs& a, int r0, int r_end, float* al)
{
    const int ty = threadIdx.x / 16;
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        const int r = r0 + RT * ty + i;
        al[i] = r < r_end ? window_coeff(a, __ldg(a.alpha + r % a.D)) : 0.0f;
    }
}

// Layers kernel (persistent over position tiles of PT): a3 into the stash
// rows (the last 64 rows of h), a3[j][pos] at h[(rows - 64 + j) * npos + pos].
template <bool TWO_D, int PT>
__global__ void __launch_bounds__(kFgThreads) filter_layers_kernel(FilterGenArgs a)
{
    grid_dependency_begin();
    select_sample(a);
    using LT = LayerTile<PT>;
    constexpr int AS = LT::AS, PPT = LT::PPT;
    extern __shared__ __align__(16) float fg_smem[];
    float* sW = fg_smem;
    float* sX = fg_smem + kFgWRegion;
    float* sY = sX + kFfnMaxIn * AS;
    float* sF = sY + kFfnWidth * AS;
    const long npos = fg_positions<TWO_D>(a);
    const long ntiles = (npos + PT - 1) / PT;
    float* stash = a.h + (long)(a.rows - kFfnWidth) * npos;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    stage_weights<TWO_D>(a, sW);
    if (a.film) stage_film(a, sF);
    for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const long p0 = tile * PT;
        layers_tile<TWO_D, PT>(a, npos, p0, sW, sX, sY, sF);   // ends with a barrier
        // stash a3: thread (ty, tx) stores its own 4 units x PPT positions
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int u = 4 * ty + i;
            const long pos = p0 + PPT * tx;
            float* dst = stash + (long)u * npos;
            if constexpr (PPT == 4) {
                if (a.vec) {
                    if (pos < npos)
                        *reinterpret_cast<float4*>(dst + pos) = *reinterpret_cast<const float4*>(sY + u * AS + 4 * tx);
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (pos + k < npos) dst[pos + k] = sY[u * AS + 4 * tx + k];
                }
            } else {
                if (pos < npos) dst[pos] = sY[u * AS + tx];
            }
        }
        __syncthreads();                                     // sX / sY reused by the next tile
    }
}

// Head kernel: rows 0 .. rows-65 as 128-row x 64 NG-position tiles (grid.y
// over row tiles), thread (ty, tx) owning rows 8 ty + i (i < 8) and
// positions 64 g + 4 tx + k (g < NG, k < 4).
template <bool TWO_D, int NG>
__global__ void __launch_bounds__(kFgThreads, NG == 1 ? 3 : 2) filter_head_kernel(FilterGenArgs a)
{
    grid_dependency_begin();
    select_sample(a);
    extern __shared__ __align__(16) float fg_smem[];
    float* sWT = fg_smem;                                   // [64][132]: Wout tile, transposed
    float* sA = fg_smem + kFfnWidth * kFgRS;                // [64][64 NG + 4]: a3 tile
    const long npos = fg_positions<TWO_D>(a);
    const long p0 = (long)blockIdx.x * (64 * NG);
    const int r0 = blockIdx.y * kFgRowTile;
    const int stash_row = a.rows - kFfnWidth;
    float al[8];
    load_alpha<8>(a, r0, stash_row, al);
    load_a3_tile<NG>(a, npos, p0, a.h + (long)stash_row * npos, sA);
    load_wout_tile<kFgRowTile, kFgRS>(a, r0, stash_row, sWT);
    __syncthreads();
    head_block<TWO_D, 8, kFgRS, NG>(a, npos, p0, r0, stash_row, sWT, sA, al);
}

// Tail kernel: the 64 stash rows for 64 positions per CTA; each CTA reads
// its own 64 x 64 tile of a3 before overwriting exactly that tile.
template <bool TWO_D>
__global__ void __launch_bounds__(kFgThreads) filter_tail_kernel(FilterGenArgs a)
{
    grid_dependency_begin();
    select_sample(a);
    extern __shared__ __align__(16) float fg_smem[];
    float* sWT = fg_smem;                                   // [64][68]: Wout stash rows, transposed
    float* sA = fg_smem + kFfnWidth * kFgUS;                // [64][68]: a3 tile
    const long npos = fg_positions<TWO_D>(a);
    const long p0 = (long)blockIdx.x * kFgTile;
    const int stash_row = a.rows - kFfnWidth;
    float al[4];
    load_alpha<4>(a, stash_row, a.rows, al);
    load_a3_tile<1>(a, npos, p0, a.h + (long)stash_row * npos, sA);
    load_wout_tile<kFfnWidth, kFgUS>(a, stash_row, a.rows, sWT);
    __syncthreads();
    head_block<TWO_D, 4, kFgUS, 1>(a, npos, p0, stash_row, a.rows, sWT, sA, al);
}

// Tail kernel for short filters: 16 positions per CTA (more CTAs), thread
// (ty, tx) owning stash rows 4 ty + i (i < 4) at position tx.
template <bool TWO_D>
__global__ void __launch_bounds__(kFgThreads) filter_tail16_kernel(FilterGenArgs a)
{
    grid_dependency_begin();
    select_sample(a);
    constexpr int PT = kFgSmallTile, AS = PT + 4;
    extern __shared__ __align__(16) float fg_smem[];
    float* sWT = fg_smem;                                   // [64][68]: Wout stash rows, transposed
    float* sA = fg_smem + kFfnWidth * kFgUS;                // [64][20]: a3 tile
    const long npos = fg_positions<TWO_D>(a);
    const long p0 = (long)blockIdx.x * PT;
    const int stash_row = a.rows - kFfnWidth;
    float* stash = a.h + (long)stash_row * npos;
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    float al[4];
    load_alpha<4>(a, stash_row, a.rows, al);
    {
        constexpr int PER = kFfnWidth * PT / kFgThreads;
        float v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = tid + i * kFgThreads, j = e / PT, pp = e % PT;
            v[i] = p0 + pp < npos ? stash[(long)j * npos + p0 + pp] : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = tid + i * kFgThreads;
            sA[(e / PT) * AS + e % PT] = v[i];
        }
    }
    load_wout_tile<kFfnWidth, kFgUS>(a, stash_row, a.rows, sWT);
    __syncthreads();
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 8
    for (int j = 0; j < kFfnWidth; ++j) {
        const float4 w = *reinterpret_cast<const float4*>(sWT + j * kFgUS + 4 * ty);
        const float x = sA[j * AS + tx];
        acc[0] = fmaf(w.x, x, acc[0]);
        acc[1] = fmaf(w.y, x, acc[1]);
        acc[2] = fmaf(w.z, x, acc[2]);
        acc[3] = fmaf(w.w, x, acc[3]);
    }
    const long pos = p0 + tx;
    if (pos >= npos) return;
    const float u = window_u<TWO_D>(a, pos);
#pragma unroll
    for (int i = 0; i < 4; ++i) stash[(long)(4 * ty + i) * npos + pos] = acc[i] * expf(al[i] * u);
}

// Single launch for at most 64 rows: every CTA evaluates the layers of its
// 64 positions, then the head for all rows from shared memory.
template <bool TWO_D>
__global__ void __launch_bounds__(kFgThreads) filter_gen_kernel(FilterGenArgs a)
{
    grid_dependency_begin();
    select_sample(a);
    using LT = LayerTile<kFgTile>;
    extern __shared__ __align__(16) float fg_smem[];
    float* sW = fg_smem;
    float* sX = fg_smem + kFgWRegion;
    float* sY = sX + kFfnMaxIn * LT::AS;
    float* sF = sY + kFfnWidth * LT::AS;
    const long npos = fg_positions<TWO_D>(a);
    const long p0 = (long)blockIdx.x * kFgTile;
    float al[4];
    load_alpha<4>(a, 0, a.rows, al);
    stage_weights<TWO_D>(a, sW);
    if (a.film) stage_film(a, sF);
    layers_tile<TWO_D, kFgTile>(a, npos, p0, sW, sX, sY, sF);  // ends with a barrier
    load_wout_tile<kFfnWidth, kFgUS>(a, 0, a.rows, sW);   // the weights are no longer read
    __syncthreads();
    static_assert(LT::AS == kFgUS, "a3 tile stride");
    head_block<TWO_D, 4, kFgUS, 1>(a, npos, p0, 0, a.rows, sW, sY, al);
}

}  // namespace hyena
