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

template <int LOG2Z2>
struct Fft3dZ {
    using FZ = SmemFft<LOG2Z2>;
    static constexpr int Z2 = 1 << LOG2Z2;              // 2Z
    static constexpr int TC = (256 / FZ::T) > 16 ? 16 : ((256 / FZ::T) < 2 ? 2 : 256 / FZ::T);
    static constexpr int THREADS = TC * FZ::T;
    static constexpr int STRIDE = stride_mod16(Z2, 16 / (TC > 16 ? 16 : TC));
    static constexpr size_t SMEM = sizeof(float2) * TC * STRIDE;
    static_assert(THREADS <= 1024 && SMEM <= 227 * 1024, "z kernel geometry");
};

// z kernel.  MODE 0 (forward): per image qi of the wave, CTAs over
// (ky, block of TC slots kx) take the z transform of kx != 0, multiply,
// and transform back (planes z < Z kept); then one CTA per pair u in
// [0, H] takes slot 0 of rows ky = u and 2H - u together.  MODE 1
// (spectra): forward z transform of every slot of the filters' planes
// z < Z, all 2Z planes written.
template <int LOG2Z2, int MODE>
__global__ void __launch_bounds__(Fft3dZ<LOG2Z2>::THREADS)
fft3d_z_kernel(Fft2dArgs a)
{
    grid_dependency_begin();
    using ZL = Fft3dZ<LOG2Z2>;
    using FZ = typename ZL::FZ;
    constexpr int Z2 = ZL::Z2, TC = ZL::TC, ZH = Z2 / 2, V = FZ::V;
    const int W = a.W, H2 = 2 * a.Hp;
    const int kxb = W / TC;                               // slot blocks per row
    const long reg_per_img = (long)H2 * kxb;              // regular CTAs per image
    extern __shared__ __align__(16) float2 smem_z[];
    const int tid = threadIdx.x;
    const int cc = tid % TC, t = tid / TC;
    float2* buf = smem_z + cc * ZL::STRIDE;
    const int pt = pad16(t);
    const size_t plane = (size_t)H2 * W;                  // slots per plane
    float2 reg[V];

    // which image and which columns this CTA takes
    const long blk = blockIdx.x;
    const bool pair_cta = MODE == 0 && blk >= (long)a.nq * reg_per_img;
    int qi, ky, kx;
    if (!pair_cta) {
        qi = (int)(blk / reg_per_img);
        const long rem = blk % reg_per_img;
        ky = (int)(rem / kxb);
        kx = (int)(rem % kxb) * TC + cc;
    } else {
        const long pb = blk - (long)a.nq * reg_per_img;
        qi = (int)(pb / (a.Hp + 1));
        const int u = (int)(pb % (a.Hp + 1));
        // columns 0 and 1: slot 0 of rows u and 2H - u (one row when they coincide)
        ky = cc == 0 ? u : (H2 - u) % H2;
        kx = 0;
    }
    const int q = a.q0 + qi;
    const size_t zplanes = MODE == 1 ? (size_t)2 * a.zp : (size_t)a.zp;   // planes allocated per image
    float2* colp = a.S + (size_t)qi * zplanes * plane + (size_t)ky * W + kx;
    // a CTA column that writes: regular columns kx != 0 (all in MODE 1),
    // and the pair CTA's first two columns (the second only if distinct)
    const bool self_pair = pair_cta && (ky == (H2 - ky) % H2);
    const bool live = !pair_cta ? (MODE == 1 || kx != 0) : (cc == 0 || (cc == 1 && !(ky == 0 || 2 * ky == H2)));

    // forward z transform of planes z < Z (zero beyond)
    static_for<V>([&](auto rr) {
        constexpr int r = decltype(rr)::value;
        const int z = t + r * (Z2 / V);
        buf[pad16_at<Z2 / V>(t, pt, r)] = (r < V / 2 && (live || pair_cta)) ? colp[(size_t)z * plane]
                                                                             : make_float2(0.0f, 0.0f);
    });
    __syncthreads();
    FZ::template run<-1, true>(buf, reg, t);
    if constexpr (MODE == 1) {
        if (live)
            static_for<V>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                colp[(size_t)(t + r * (Z2 / V)) * plane] = reg[r];
            });
        return;
    } else {
        static_for<V>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            buf[pad16_at<Z2 / V>(t, pt, r)] = reg[r];
        });
        __syncthreads();
        const int c = q / a.B;
        const float bias = __ldg(a.bias + a.n * a.C + c);
        const float2* Hn = a.Hs + ((size_t)a.n * a.C + c) * Z2 * plane;   // [2Z][2H][W]
        const float s = 1.0f / ((float)Z2 * (float)H2);
        if (!pair_cta) {
            if (live)
                static_for<V>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    const int kz = t + r * (Z2 / V);
                    const float2 hv = __ldg(Hn + (size_t)kz * plane + (size_t)ky * W + kx);
                    const int pk = pad16_at<Z2 / V>(t, pt, r);
                    buf[pk] = cmul(buf[pk], make_float2((hv.x + bias) * s, hv.y * s));
                });
        } else {
            // slot 0: column 0 (row u) pairs with column 1 (row 2H - u, or
            // itself when u = 0 or H) at kz' = -kz
            float2* bA = smem_z;                                // column 0
            float2* bB = self_pair ? smem_z : smem_z + ZL::STRIDE;
            const int u = ky;                                   // the first column's row (cc == 0 threads)
            const int u2 = (H2 - u) % H2;
            const int nkz = self_pair ? ZH + 1 : Z2;
            if (cc == 0) {
                for (int kz = t; kz < nkz; kz += FZ::T) {
                    const int kz2 = (Z2 - kz) % Z2;
                    const float2 A = bA[pad16(kz)], Bp = bB[pad16(kz2)];
                    const float2 p1 = __ldg(Hn + (size_t)kz * plane + (size_t)u * W);
                    const float2 p2 = __ldg(Hn + (size_t)kz2 * plane + (size_t)u2 * W);
                    // X0 = (A + conj B')/2, XW = (A - conj B')/(2i); the filter likewise
                    const float2 x0 = make_float2(0.5f * (A.x + Bp.x), 0.5f * (A.y - Bp.y));
                    const float2 xw = make_float2(0.5f * (A.y + Bp.y), -0.5f * (A.x - Bp.x));
                    const float2 h0 = make_float2(0.5f * (p1.x + p2.x) + bias, 0.5f * (p1.y - p2.y));
                    const float2 hw = make_float2(0.5f * (p1.y + p2.y) + bias, -0.5f * (p1.x - p2.x));
                    const float2 y0 = cmul(x0, h0), yw = cmul(xw, hw);
                    // (kz, u): Y0 + i YW;  (-kz, 2H - u): conj(Y0) + i conj(YW)
                    const float2 nA = make_float2(s * (y0.x - yw.y), s * (y0.y + yw.x));
                    const float2 nB = make_float2(s * (y0.x + yw.y), s * (yw.x - y0.y));
                    if (self_pair && kz2 < kz) continue;        // handled from the partner
                    if (!(self_pair && kz2 == kz)) bB[pad16(kz2)] = nB;
                    bA[pad16(kz)] = nA;
                }
            }
        }
        __syncthreads();
        FZ::template run<+1, true>(buf, reg, t);
        if (live)
            static_for<V / 2>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                colp[(size_t)(t + r * (Z2 / V)) * plane] = reg[r];
            });
    }
}

}  // namespace hyena
