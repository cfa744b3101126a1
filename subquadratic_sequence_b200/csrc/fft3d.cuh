// fft3d.cuh -- the 3-D Hyena forward and 3-D filter spectra: the z axis.
//
// Per image (b, c) and order n: the linear 3-D convolution of z_{n-1}
// [Z][H][W] with h_n [Z][H][W] (offsets 0..Z-1 x 0..H-1 x 0..W-1) through
// the 3-D DFT of the volume zero-padded to 2Z x 2H x 2W ("Native
// Multi-Dimensional Subquadratic Operators via Input Dependent Long
// Convolutions": Native ND Convolution on N-dimensional grids, Handling
// Boundaries), plus the bias, cropped and gated -- the same recurrence.
//
// Each z-plane goes through the 2-D machinery: the packed row transform
// (slot 0 holding bins 0 and W of the row as one complex number) and the
// 2H-point column transform, planes kept at a pitch of 2H rows.  This file
// adds the 2Z-point transform along z of every slot (ky, kx), the spectral
// multiply, and its inverse.  Slot 0 carries A = X0 + i XW, two transforms
// of real volumes, so its bins pair across (kz, ky) and (-kz, -ky):
//     X0 = (A + conj A') / 2,   XW = (A - conj A') / (2 i),
// A' the value at (-kz, -ky); each is multiplied by its own filter part
// plus the bias and the pair is re-packed.  One order is: z kernel, inverse
// columns (rows y < H), inverse rows with the gate and the next order's
// forward rows, forward columns.
#pragma once

#include "fft2d.cuh"

namespace hyena {

template <int LOG2Z2, bool PAD = true>
struct Fft3dZ {
    using FZ = SmemFft<LOG2Z2>;
    static constexpr int Z2 = 1 << LOG2Z2;              // transform length: 2Z (padded) or Z (circular)
    static constexpr int TC = (256 / FZ::T) > 16 ? 16 : ((256 / FZ::T) < 2 ? 2 : 256 / FZ::T);
    static constexpr int THREADS = TC * FZ::T;
    static constexpr int STRIDE = stride_mod16(Z2, 16 / (TC > 16 ? 16 : TC));
    static constexpr size_t SMEM = sizeof(float2) * TC * STRIDE;
    // resident CTAs per SM the register budget aims at: 96 registers a
    // thread (128 for one-warp CTAs and for circular transforms, whose
    // whole column is live; no cap with 32 values a thread).  Registers are
    // allocated per warp.
    static constexpr int REGS = (THREADS < 64 || !PAD) ? 128 : 96;
    static constexpr int WARP_THREADS = (THREADS + 31) / 32 * 32;
    static constexpr int MIN_BLOCKS = FZ::V == 32 ? 1 : 65536 / (WARP_THREADS * REGS);
    static_assert(THREADS <= 1024 && SMEM <= 227 * 1024, "z kernel geometry");
};

// z kernel.  MODE 0 (forward): CTAs per channel of the wave over (ky,
// block of TC slots kx) hold the channel's filter column (the 2Z spectrum
// values of their slots, bias and scale folded in) in registers and apply
// it to every volume of that channel in the wave: z transform, multiply,
// inverse, planes z < Z kept.  kx = 0 is left to the pair CTAs: each takes
// TC/2 pairs u in [0, H], slot 0 of rows ky = u (column 2j) and 2H - u
// (column 2j + 1).  MODE 2: MODE 0 with per-sample spectra, each volume b
// of the channel loading sample b's column (at Hs + b Hs_bstride) instead.
// MODE 1 (spectra): forward z transform of every slot of
// the filters' planes z < Z, all 2Z planes written.  Circular (PAD false):
// Z-point transforms of all Z planes, H rows a plane, nothing cropped.
template <int LOG2Z2, int MODE, bool PAD = true>
__global__ void __launch_bounds__(Fft3dZ<LOG2Z2, PAD>::THREADS, Fft3dZ<LOG2Z2, PAD>::MIN_BLOCKS)
fft3d_z_kernel(Fft2dArgs a)
{
    grid_dependency_begin();
    using ZL = Fft3dZ<LOG2Z2, PAD>;
    using FZ = typename ZL::FZ;
    constexpr int Z2 = ZL::Z2, TC = ZL::TC, ZH = Z2 / 2, V = FZ::V, NP = TC / 2;
    constexpr int VL = PAD ? V / 2 : V;                   // registers holding grid planes
    const int W = a.W, H2 = (PAD ? 2 : 1) * a.Hp;       // slots per row, rows per plane
    const int UH = H2 / 2;                                // slot-0 pairs u in [0, UH]
    const int kxb = W / TC;                               // slot blocks per row
    const long reg_per = (long)H2 * kxb;                  // regular CTAs per image / channel
    extern __shared__ __align__(16) float2 smem_z[];
    const int tid = threadIdx.x;
    const int cc = tid % TC, t = tid / TC;
    float2* buf = smem_z + cc * ZL::STRIDE;
    const int pt = pad16(t);
    const size_t plane = (size_t)H2 * W;                  // slots per plane
    const long blk = blockIdx.x;
    float2 reg[V];

    // the grid planes of a slot column into the buffer (padded: the upper
    // half is zero padding, which the forward transform does not read)
    auto load_col = [&](const float2* colp) {
        static_for<VL>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            buf[pad16_at<Z2 / V>(t, pt, r)] = colp[(size_t)(t + r * (Z2 / V)) * plane];
        });
        __syncthreads();
    };

    if constexpr (MODE == 1) {
        const int qi = (int)(blk / reg_per);
        const long rem = blk % reg_per;
        const int ky = (int)(rem / kxb), kx = (int)(rem % kxb) * TC + cc;
        float2* colp = a.S + (size_t)qi * Z2 * plane + (size_t)ky * W + kx;
        load_col(colp);
        FZ::template run<-1, true, PAD>(buf, reg, t);
        static_for<V>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            colp[(size_t)(t + r * (Z2 / V)) * plane] = reg[r];
        });
        return;
    } else {
        const int cfirst = a.q0 / a.B;
        const int nch = (a.q0 + a.nq - 1) / a.B - cfirst + 1;
        const bool pair_cta = blk >= (long)nch * reg_per;
        const int npair = (UH + 1 + NP - 1) / NP;         // pair CTAs per channel
        int ci, ky, kx;
        bool live;
        int u = 0;
        if (!pair_cta) {
            ci = (int)(blk / reg_per);
            const long rem = blk % reg_per;
            ky = (int)(rem / kxb);
            kx = (int)(rem % kxb) * TC + cc;
            live = kx != 0;
        } else {
            const long pb = blk - (long)nch * reg_per;
            ci = (int)(pb / npair);
            u = (int)(pb % npair) * NP + cc / 2;          // this column's pair
            const bool valid = u <= UH;
            const int uu = valid ? u : UH;
            const bool self = uu == 0 || uu == UH;        // rows u and H2 - u coincide
            ky = (cc % 2 == 0) ? uu : (H2 - uu) % H2;
            kx = 0;
            live = valid && (cc % 2 == 0 || !self);
        }
        const int c = cfirst + ci;
        const int qa = max(a.q0, c * a.B), qb = min(a.q0 + a.nq, (c + 1) * a.B);
        const float bias = __ldg(a.bias + a.n * a.C + c);
        const float2* Hn = a.Hs + ((size_t)a.n * a.C + c) * Z2 * plane;   // [2Z][2H][W]
        // per-sample spectra (MODE 2): volume q = c B + b takes sample b's set.
        // The mode is a template parameter, so the shared kernel carries no
        // branch; inside MODE 2 the branch stays a run-time one, which measured
        // faster than the compile-time form (that one lets the compiler move the
        // next volume's filter loads ahead and spill)
        const bool ps = MODE == 2 && a.Hs_bstride != 0;
        auto spectra_of = [&](int q) { return ps ? Hn + (size_t)(q - c * a.B) * a.Hs_bstride : Hn; };
        const float s = 1.0f / ((float)Z2 * (float)H2);
        if (!pair_cta) {
            // the filter column, (H + b) / (2Z 2H), in register order; loaded
            // once for the channel, or per volume with per-sample spectra
            float2 hv[V];
            auto load_filter = [&](const float2* Hq) {
                static_for<V>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    const float2 h = __ldg(Hq + (size_t)(t + r * (Z2 / V)) * plane + (size_t)ky * W + kx);
                    hv[r] = make_float2((h.x + bias) * s, h.y * s);
                });
            };
            if (!ps) load_filter(Hn);
            for (int q = qa; q < qb; ++q) {
                if (ps) load_filter(spectra_of(q));
                float2* colp = a.S + (size_t)(q - a.q0) * a.zp * plane + (size_t)ky * W + kx;
                load_col(colp);
                FZ::template run<-1, true, PAD>(buf, reg, t);
                static_for<V>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    buf[pad16_at<Z2 / V>(t, pt, r)] = cmul(reg[r], hv[r]);
                });
                __syncthreads();
                FZ::template run<+1, true>(buf, reg, t);
                if (live)
                    static_for<VL>([&](auto rr) {
                        constexpr int r = decltype(rr)::value;
                        colp[(size_t)(t + r * (Z2 / V)) * plane] = reg[r];
                    });
            }
        } else {
            const int u0 = (int)((blk - (long)nch * reg_per) % npair) * NP;
            for (int q = qa; q < qb; ++q) {
                const float2* Hq = spectra_of(q);
                float2* colp = a.S + (size_t)(q - a.q0) * a.zp * plane + (size_t)ky * W;
                load_col(colp);
                FZ::template run<-1, true, PAD>(buf, reg, t);
                static_for<V>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    buf[pad16_at<Z2 / V>(t, pt, r)] = reg[r];
                });
                __syncthreads();
                // slot 0 of pair j: column 2j (row u) with column 2j + 1
                // (row 2H - u, or column 2j itself when u = 0 or H) at kz' = -kz
                for (int e = tid; e < NP * Z2; e += ZL::THREADS) {
                    const int j = e / Z2, kz = e % Z2;
                    const int uj = u0 + j;
                    const bool self = uj == 0 || uj == UH;
                    if (uj > UH || (self && kz > ZH)) continue;
                    const int u2 = (H2 - uj) % H2;
                    float2* bA = smem_z + (2 * j) * ZL::STRIDE;
                    float2* bB = self ? bA : smem_z + (2 * j + 1) * ZL::STRIDE;
                    const int kz2 = (Z2 - kz) % Z2;
                    const float2 A = bA[pad16(kz)], Bp = bB[pad16(kz2)];
                    const float2 p1 = __ldg(Hq + (size_t)kz * plane + (size_t)uj * W);
                    const float2 p2 = __ldg(Hq + (size_t)kz2 * plane + (size_t)u2 * W);
                    // X0 = (A + conj B')/2, XW = (A - conj B')/(2i); the filter likewise
                    const float2 x0 = make_float2(0.5f * (A.x + Bp.x), 0.5f * (A.y - Bp.y));
                    const float2 xw = make_float2(0.5f * (A.y + Bp.y), -0.5f * (A.x - Bp.x));
                    const float2 h0 = make_float2(0.5f * (p1.x + p2.x) + bias, 0.5f * (p1.y - p2.y));
                    const float2 hw = make_float2(0.5f * (p1.y + p2.y) + bias, -0.5f * (p1.x - p2.x));
                    const float2 y0 = cmul(x0, h0), yw = cmul(xw, hw);
                    // (kz, u): Y0 + i YW;  (-kz, 2H - u): conj(Y0) + i conj(YW)
                    bA[pad16(kz)] = make_float2(s * (y0.x - yw.y), s * (y0.y + yw.x));
                    if (!(self && kz2 == kz)) bB[pad16(kz2)] = make_float2(s * (y0.x + yw.y), s * (yw.x - y0.y));
                }
                __syncthreads();
                FZ::template run<+1, true>(buf, reg, t);
                if (live)
                    static_for<VL>([&](auto rr) {
                        constexpr int r = decltype(rr)::value;
                        colp[(size_t)(t + r * (Z2 / V)) * plane] = reg[r];
                    });
            }
        }
    }
}

}  // namespace hyena
