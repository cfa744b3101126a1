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
// One CTA takes TILE consecutive positions: TILE threads evaluate the
// three sine layers (one position each, weights broadcast from shared
// memory), then all threads run the head as a TILE x 64 by 64 x rows
// product out of shared memory and write h coalesced along the position.
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
constexpr int kFgThreads = 256;
// dynamic shared memory: W1 [64][66], W2, W3 [64][64] (the head's Wout
// chunk [64][65] reuses this region afterwards), then a3 [64][TILE+1]
constexpr int kFgWRegion = kFfnWidth * kFfnMaxIn + 2 * kFfnWidth * kFfnWidth;
constexpr size_t kFgSmemBytes = sizeof(float) * (kFgWRegion + kFfnWidth * (kFgTile + 1));

template <bool TWO_D>
__global__ void __launch_bounds__(kFgThreads) filter_gen_kernel(FilterGenArgs a)
{
    extern __shared__ __align__(16) float fg_smem[];
    float* sW1 = fg_smem;                                   // [64][66]
    float* sW2 = sW1 + kFfnWidth * kFfnMaxIn;               // [64][64]
    float* sW3 = sW2 + kFfnWidth * kFfnWidth;               // [64][64]
    float* sOut = fg_smem;                                  // [64][65], after the layers
    float* sAct = fg_smem + kFgWRegion;                     // [64][TILE+1]
    constexpr int AS = kFgTile + 1;

    const int tid = threadIdx.x;
    const long npos = TWO_D ? (long)a.Hh * a.Ww : (long)a.L;
    const long p0 = (long)blockIdx.x * kFgTile;

    // weights into shared memory, zero padded to 64 x 64 (sin(0) = 0, so
    // padded units contribute nothing)
    // W1's columns go to a canonical layout in which every feature has a
    // fixed slot: 1-D [t, (sin, cos) band 1..16]; 2-D [ty, tx, (sin, cos)
    // y-band 1..16, (sin, cos) x-band 1..16].
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
        sW1[e] = (r < a.width && src >= 0) ? __ldg(a.W1 + r * a.n_in + src) : 0.0f;
    }
    for (int e = tid; e < kFfnWidth * kFfnWidth; e += kFgThreads) {
        const int r = e / kFfnWidth, c = e % kFfnWidth;
        const bool in = r < a.width && c < a.width;
        sW2[e] = in ? __ldg(a.W2 + r * a.width + c) : 0.0f;
        sW3[e] = in ? __ldg(a.W3 + r * a.width + c) : 0.0f;
    }
    __syncthreads();

    if (tid < kFgTile) {
        const long pos = min(p0 + tid, npos - 1);
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
                float s, c;
                sincospif(2.0f * (float)qk / (float)a.L, &s, &c);
                phi[2 * k - 1] = s;
                phi[2 * k] = c;
            }
        } else {
            const int iy = (int)(pos / a.Ww), ix = (int)(pos % a.Ww);
            phi[0] = (float)iy / (float)a.Hh;
            phi[1] = (float)ix / (float)a.Ww;
#pragma unroll
            for (int k = 1; k <= (kFfnMaxIn - 2) / 4; ++k) {
                if (k > a.n_bands) break;
                float s, c;
                const int qy = (int)(((long)k * iy) % a.Hh);
                sincospif(2.0f * (float)qy / (float)a.Hh, &s, &c);
                phi[2 * k] = s;
                phi[2 * k + 1] = c;
            }
#pragma unroll
            for (int k = 1; k <= (kFfnMaxIn - 2) / 4; ++k) {
                if (k > a.n_bands) break;
                float s, c;
                const int qx = (int)(((long)k * ix) % a.Ww);
                sincospif(2.0f * (float)qx / (float)a.Ww, &s, &c);
                phi[2 + 2 * 16 + 2 * (k - 1)] = s;
                phi[2 + 2 * 16 + 2 * (k - 1) + 1] = c;
            }
        }
        // layer 1 (outputs staged in this thread's column of sAct)
#pragma unroll 1
        for (int j = 0; j < kFfnWidth; ++j) {
            float s = 0.0f;
#pragma unroll
            for (int c = 0; c < kFfnMaxIn; ++c) s = fmaf(sW1[j * kFfnMaxIn + c], phi[c], s);
            sAct[j * AS + tid] = sinf(s);
        }
        // layers 2 and 3
#pragma unroll 1
        for (int layer = 0; layer < 2; ++layer) {
            const float* Wl = layer == 0 ? sW2 : sW3;
            float act[kFfnWidth];
#pragma unroll
            for (int c = 0; c < kFfnWidth; ++c) act[c] = sAct[c * AS + tid];
#pragma unroll 1
            for (int j = 0; j < kFfnWidth; ++j) {
                float s = 0.0f;
#pragma unroll
                for (int c = 0; c < kFfnWidth; ++c) s = fmaf(Wl[j * kFfnWidth + c], act[c], s);
                sAct[j * AS + tid] = sinf(s);
            }
        }
    }
    __syncthreads();

    // head: out[r][p] = sum_j Wout[r][j] a3[j][p], times the window.
    // Thread (ty, tx) of a 16 x 16 grid computes rows ty + 16 i and
    // positions tx + 16 k (i, k < 4) of each 64 x 64 tile.
    const int tx = tid % 16, ty = tid / 16;
    constexpr int OS = kFfnWidth + 1;
    for (int r0 = 0; r0 < a.rows; r0 += kFgTile) {
        __syncthreads();
        for (int e = tid; e < kFgTile * kFfnWidth; e += kFgThreads) {
            const int r = e / kFfnWidth, j = e % kFfnWidth;
            sOut[r * OS + j] = (r0 + r < a.rows && j < a.width)
                                   ? __ldg(a.Wout + (long)(r0 + r) * a.width + j) : 0.0f;
        }
        __syncthreads();
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[i][k] = 0.0f;
#pragma unroll 8
        for (int j = 0; j < kFfnWidth; ++j) {
            float w[4], x[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = sOut[(ty + 16 * i) * OS + j];
#pragma unroll
            for (int k = 0; k < 4; ++k) x[k] = sAct[j * AS + tx + 16 * k];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[i][k] = fmaf(w[i], x[k], acc[i][k]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
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
}

}  // namespace hyena
