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
// One CTA takes a tile of 64 consecutive positions and up to 128 head rows
// (a 2-D grid: position tiles x row tiles).  All 256 threads evaluate the
// three sine layers -- four threads per position, 16 output units each, so
// every thread runs 16 independent accumulation chains -- with weights and
// activations in shared memory; then the head runs as a 64-position x
// 128-row x 64 product out of shared memory and h is written coalesced
// along the position.  The layers are recomputed by every row tile of a
// position tile: 64 x 9.3k multiply-adds, cheaper than a scratch round trip.
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

constexpr int kFgTile = 64;        // positions per CTA
constexpr int kFgRowTile = 128;    // head rows per CTA
constexpr int kFgThreads = 256;
constexpr int kFgAS = kFgTile + 1; // activation row stride
constexpr int kFgOS = kFfnWidth + 1;
// weight row strides: odd, so the four units a position's threads read at
// once (rows 4 jj + q, q < 4) sit on four different banks
constexpr int kFgW1S = kFfnMaxIn + 1;
constexpr int kFgWS = kFfnWidth + 1;
// dynamic shared memory (floats): W1 [64][67], W2, W3 [64][65], two
// activation buffers [64][65]; the head's Wout tile [128][65] reuses the
// weight region
constexpr int kFgWRegion = kFfnWidth * kFgW1S + 2 * kFfnWidth * kFgWS;
static_assert(kFgRowTile * kFgOS <= kFgWRegion, "Wout tile fits the weight region");
constexpr size_t kFgSmemBytes = sizeof(float) * (kFgWRegion + 2 * kFfnWidth * kFgAS);

template <bool TWO_D>
__global__ void __launch_bounds__(kFgThreads) filter_gen_kernel(FilterGenArgs a)
{
    extern __shared__ __align__(16) float fg_smem[];
    float* sW1 = fg_smem;                                   // [64][67]
    float* sW2 = sW1 + kFfnWidth * kFgW1S;                  // [64][65]
    float* sW3 = sW2 + kFfnWidth * kFgWS;                   // [64][65]
    float* sOut = fg_smem;                                  // [128][65], after the layers
    float* sA = fg_smem + kFgWRegion;                       // [64][65]  a1, a3
    float* sB = sA + kFfnWidth * kFgAS;                     // [64][65]  a2

    const int tid = threadIdx.x;
    const long npos = TWO_D ? (long)a.Hh * a.Ww : (long)a.L;
    const long p0 = (long)blockIdx.x * kFgTile;
    const int r0 = blockIdx.y * kFgRowTile;

    // W1's columns go to a canonical layout in which every feature has a
    // fixed slot: 1-D [t, (sin, cos) band 1..16]; 2-D [ty, tx, (sin, cos)
    // y-band 1..16, (sin, cos) x-band 1..16].  Units beyond `width` are
    // zero: sin(0) = 0, so they contribute nothing.
    for (int e = tid; e < kFfnWidth * kFfnMaxIn; e += kFgThreads) {
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
    for (int e = tid; e < kFfnWidth * kFfnWidth; e += kFgThreads) {
        const int r = e / kFfnWidth, c = e % kFfnWidth;
        const bool in = r < a.width && c < a.width;
        sW2[r * kFgWS + c] = in ? __ldg(a.W2 + r * a.width + c) : 0.0f;
        sW3[r * kFgWS + c] = in ? __ldg(a.W3 + r * a.width + c) : 0.0f;
    }

    // ---- three sine layers: thread (p, q) computes units 4 jj + q
    // (jj < 16) of position p0 + p
    const int p = tid / 4, q = tid % 4;
    {
        const long pos = min(p0 + p, npos - 1);
        float phi[kFfnMaxIn];
#pragma unroll
        for (int c = 0; c < kFfnMaxIn; ++c) phi[c] = 0.0f;
        if constexpr (!TWO_D) {
            const int i = (int)pos;
            phi[0] = (float)i / (float)a.L;
#pragma unroll
            for (int k = 1; k <= (kFfnMaxIn - 1) / 2; ++k) {
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
            for (int k = 1; k <= (kFfnMaxIn - 2) / 4; ++k) {
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
        __syncthreads();                                   // weights staged
        float acc[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) acc[jj] = 0.0f;
#pragma unroll
        for (int c = 0; c < kFfnMaxIn; ++c)
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
                acc[jj] = fmaf(sW1[(4 * jj + q) * kFgW1S + c], phi[c], acc[jj]);
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) sA[(4 * jj + q) * kFgAS + p] = sinf(acc[jj]);
    }
    __syncthreads();
#pragma unroll 1
    for (int layer = 0; layer < 2; ++layer) {
        const float* Wl = layer == 0 ? sW2 : sW3;
        const float* in = layer == 0 ? sA : sB;
        float* out = layer == 0 ? sB : sA;
        float acc[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) acc[jj] = 0.0f;
#pragma unroll 8
        for (int c = 0; c < kFfnWidth; ++c) {
            const float x = in[c * kFgAS + p];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) acc[jj] = fmaf(Wl[(4 * jj + q) * kFgWS + c], x, acc[jj]);
        }
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) out[(4 * jj + q) * kFgAS + p] = sinf(acc[jj]);
        __syncthreads();
    }

    // ---- head: out[r][p] = sum_j Wout[r][j] a3[j][p], times the window.
    // Thread (ty, tx) of a 16 x 16 grid computes rows ty + 16 i (i < 8) and
    // positions tx + 16 k (k < 4).
    for (int e = tid; e < kFgRowTile * kFfnWidth; e += kFgThreads) {
        const int r = e / kFfnWidth, j = e % kFfnWidth;
        sOut[r * kFgOS + j] = (r0 + r < a.rows && j < a.width)
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
        if (r >= a.rows) continue;
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

}  // namespace hyena
