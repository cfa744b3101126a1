// fft3d_bwd.cuh -- the backward pass of the 3-D recurrence: the z axis.
//
// The pages describe the forward only; its gradient is the chain rule on
// the 3-D linear convolution through the grid padded to 2Z x 2H x 2W
// ("Native Multi-Dimensional Subquadratic Operators via Input Dependent
// Long Convolutions": Native ND Convolution, Handling Boundaries), the
// same algebra as in 1-D and 2-D.  With c_n = h_n (*) z_n + b_n z_n,
// z_{n+1} = x_n c_n and g = dL/dz_{n+1}:
//     dx_n = g c_n,  e = g x_n,  dh_n += E conj(Z_n),  db_n = dh_n[0][0][0],
//     g <- IDFT((conj(H_n) + b_n) E), planes z < Z, rows y < H, columns x < W.
//
// The rows and columns of every plane are the 2-D backward's and the 2-D
// column kernels' work (planes at a pitch of 2H rows in the scratch); this
// file adds the z step.  Per wave of volumes:
//   A. the forward again, with the z kernel (MODE 0) saving each volume's
//      3-D spectrum Z_n (all 2Z planes) before the multiply by H_n + b_n;
//   B. per order n = N-1 .. 0: rows (g, dx_n, e, forward rows of e),
//      forward columns, the z kernel (MODE 1): forward z transform of E,
//      dh spectrum += E conj(Z_n), multiply by conj(H_n) + b_n, inverse z
//      transform, planes z < Z back; inverse columns;
//   then the inverse rows give dv.
// After the last wave the accumulated spectra go through the inverse z
// transform (MODE 2, planes z < Z kept in place), the inverse columns of
// those planes and the inverse rows: dh_n, and db_n = dh_n[0][0][0].
//
// Slot 0 of a row spectrum packs bins 0 and W of the row transform as one
// complex number, A = X0 + i XW with X0, XW the transforms of two real
// volumes; its bins pair across (kz, ky) and (-kz, -ky).  The pair CTAs
// separate both factors of every product through that pair, as the
// forward's z kernel does for the filter multiply:
//     X0 = (A + conj A') / 2,   XW = (A - conj A') / (2 i),
// and re-pack the products.  The accumulated spectrum is kept in the same
// packed form, so its inverse transforms are the plain ones.
#pragma once

#include "fft2d_bwd.cuh"
#include "fft3d.cuh"

namespace hyena {

// z kernel of the backward.  MODE 0 (A) and MODE 1 (B): the forward z
// kernel's CTAs (per channel of the wave and (ky, block of TC slots), plus
// the slot-0 pair CTAs) over the channel's volumes in the wave; MODE 0
// saves the spectrum and multiplies by (H_n + b_n), MODE 1 accumulates
// E conj(Z_n) into the channel's (or, with per-sample spectra, the
// volume's) dh spectrum and multiplies by (conj(H_n) + b_n).  MODE 2:
// inverse z transform of the accumulated spectra, one CTA per (filter,
// ky, block of slots), scaled by 1 / (2Z 2H), planes z < Z back in place.
// The volume loop is a run-time loop and so are the multiply sweeps of
// MODE 1 (four planes at a time, loads before stores), as in the 2-D
// backward's column kernel.
template <int LOG2Z2, int MODE, bool PAD = true>
__global__ void __launch_bounds__(Fft3dZ<LOG2Z2, PAD>::THREADS, Fft3dZ<LOG2Z2, PAD>::MIN_BLOCKS)
fft3d_bwd_z_kernel(Bwd2dArgs ba)
{
    grid_dependency_begin();
    const Fft2dArgs& a = ba.f;
    using ZL = Fft3dZ<LOG2Z2, PAD>;
    using FZ = typename ZL::FZ;
    constexpr int Z2 = ZL::Z2, TC = ZL::TC, ZH = Z2 / 2, V = FZ::V, NP = TC / 2;
    constexpr int VL = PAD ? V / 2 : V;                   // registers holding grid planes
    const int W = a.W, H2 = (PAD ? 2 : 1) * a.Hp;       // slots per row, rows per plane
    const int UH = H2 / 2;
    const int kxb = W / TC;
    const long reg_per = (long)H2 * kxb;
    extern __shared__ __align__(16) float2 smem_zb[];
    const int tid = threadIdx.x;
    const int cc = tid % TC, t = tid / TC;
    float2* buf = smem_zb + cc * ZL::STRIDE;
    const int pt = pad16(t);
    const size_t plane = (size_t)H2 * W;                  // slots per plane
    const size_t vol = (size_t)Z2 * plane;                // spectrum slots per volume
    const long blk = blockIdx.x;
    const float s = 1.0f / ((float)Z2 * (float)H2);
    float2 reg[V];

    if constexpr (MODE == 2) {
        const long unit = blk / reg_per, rem = blk % reg_per;
        const int ky = (int)(rem / kxb), kx = (int)(rem % kxb) * TC + cc;
        float2* colp = ba.acc + (size_t)unit * vol + (size_t)ky * W + kx;
        static_for<V>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            buf[pad16_at<Z2 / V>(t, pt, r)] = colp[(size_t)(t + r * (Z2 / V)) * plane];
        });
        __syncthreads();
        FZ::template run<+1, true>(buf, reg, t);
        static_for<VL>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            colp[(size_t)(t + r * (Z2 / V)) * plane] = make_float2(reg[r].x * s, reg[r].y * s);
        });
        return;
    } else {
        const int cfirst = a.q0 / a.B;
        const int nch = (a.q0 + a.nq - 1) / a.B - cfirst + 1;
        const bool pair_cta = blk >= (long)nch * reg_per;
        const int npair = (UH + 1 + NP - 1) / NP;
        int ci, ky, kx, u0 = 0;
        bool live;
        if (!pair_cta) {
            ci = (int)(blk / reg_per);
            const long rem = blk % reg_per;
            ky = (int)(rem / kxb);
            kx = (int)(rem % kxb) * TC + cc;
            live = kx != 0;                                // slot 0 belongs to the pair CTAs
        } else {
            const long pb = blk - (long)nch * reg_per;
            ci = (int)(pb / npair);
            u0 = (int)(pb % npair) * NP;
            const int u = u0 + cc / 2;
            const bool valid = u <= UH;
            const int uu = valid ? u : UH;
            const bool self = uu == 0 || uu == UH;
            ky = (cc % 2 == 0) ? uu : (H2 - uu) % H2;
            kx = 0;
            live = valid && (cc % 2 == 0 || !self);
        }
        const int c = cfirst + ci;
        const int qa = max(a.q0, c * a.B), qb = min(a.q0 + a.nq, (c + 1) * a.B);
        const float bias = __ldg(a.bias + a.n * a.C + c);
        const bool ps = a.Hs_bstride != 0;
        // the forward multiplies by H + b, the backward by conj(H) + b
        constexpr float cj = MODE == 0 ? 1.0f : -1.0f;
#pragma unroll 1
        for (int q = qa; q < qb; ++q) {
            const int qi = q - a.q0;
            const size_t sb = ps ? (size_t)(q - c * a.B) : 0;
            const float2* Hq = a.Hs + sb * a.Hs_bstride + ((size_t)a.n * a.C + c) * vol;
            float2* accq = ba.acc + ((sb * ba.N + a.n) * a.C + c) * vol;
            float2* zsq = ba.zsave + ((size_t)a.n * ba.wcap + qi) * vol;
            float2* colp = a.S + (size_t)qi * a.zp * plane + (size_t)ky * W + kx;
            static_for<VL>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                buf[pad16_at<Z2 / V>(t, pt, r)] = colp[(size_t)(t + r * (Z2 / V)) * plane];
            });
            __syncthreads();
            FZ::template run<-1, true, PAD>(buf, reg, t);
            if (MODE == 0 && live)
                static_for<V>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    zsq[(size_t)(t + r * (Z2 / V)) * plane + (size_t)ky * W + kx] = reg[r];
                });
            static_for<V>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                buf[pad16_at<Z2 / V>(t, pt, r)] = reg[r];
            });
            __syncthreads();
            if (!pair_cta) {
                const float2* Hc = Hq + (size_t)ky * W + kx;
                float2* ac = accq + (size_t)ky * W + kx;
                const float2* zc = zsq + (size_t)ky * W + kx;
                constexpr int K = 4;
                static_assert(V % K == 0, "plane groups");
#pragma unroll 1
                for (int r0 = 0; r0 < V; r0 += K) {
                    float2 ev[K], hv[K], zv[K], av[K];
                    static_for<K>([&](auto jj) {
                        constexpr int j = decltype(jj)::value;
                        const int kz = t + (r0 + j) * (Z2 / V);
                        ev[j] = buf[pad16(kz)];
                        hv[j] = __ldg(Hc + (size_t)kz * plane);
                        if (MODE == 1 && live) {
                            zv[j] = zc[(size_t)kz * plane];
                            av[j] = ac[(size_t)kz * plane];
                        }
                    });
                    static_for<K>([&](auto jj) {
                        constexpr int j = decltype(jj)::value;
                        const int kz = t + (r0 + j) * (Z2 / V);
                        if (MODE == 1 && live) ac[(size_t)kz * plane] = cadd(av[j], cmulc(ev[j], zv[j]));
                        buf[pad16(kz)] = cmul(ev[j], make_float2((hv[j].x + bias) * s, cj * hv[j].y * s));
                    });
                }
            } else {
                // slot 0 of pair j: column 2j (row u) with column 2j + 1 (row
                // 2H - u, or column 2j itself when u = 0 or H) at kz' = -kz
#pragma unroll 1
                for (int e = tid; e < NP * Z2; e += ZL::THREADS) {
                    const int j = e / Z2, kz = e % Z2;
                    const int uj = u0 + j;
                    const bool self = uj == 0 || uj == UH;
                    if (uj > UH || (self && kz > ZH)) continue;
                    const int u2 = (H2 - uj) % H2;
                    float2* bA = smem_zb + (2 * j) * ZL::STRIDE;
                    float2* bB = self ? bA : smem_zb + (2 * j + 1) * ZL::STRIDE;
                    const int kz2 = (Z2 - kz) % Z2;
                    const bool mirror = !(self && kz2 == kz);    // (kz2, u2) is another bin
                    const size_t i1 = (size_t)kz * plane + (size_t)uj * W;
                    const size_t i2 = (size_t)kz2 * plane + (size_t)u2 * W;
                    const float2 A = bA[pad16(kz)], Bp = bB[pad16(kz2)];
                    const float2 x0 = make_float2(0.5f * (A.x + Bp.x), 0.5f * (A.y - Bp.y));
                    const float2 xw = make_float2(0.5f * (A.y + Bp.y), -0.5f * (A.x - Bp.x));
                    if constexpr (MODE == 1) {
                        const float2 z1 = zsq[i1], z2 = zsq[i2];
                        const float2 z0 = make_float2(0.5f * (z1.x + z2.x), 0.5f * (z1.y - z2.y));
                        const float2 zw = make_float2(0.5f * (z1.y + z2.y), -0.5f * (z1.x - z2.x));
                        const float2 p0 = cmulc(x0, z0), pw = cmulc(xw, zw);
                        // (kz, u): P0 + i PW;  (-kz, 2H - u): conj(P0) + i conj(PW)
                        accq[i1] = cadd(accq[i1], make_float2(p0.x - pw.y, p0.y + pw.x));
                        if (mirror) accq[i2] = cadd(accq[i2], make_float2(p0.x + pw.y, pw.x - p0.y));
                    }
                    const float2 p1 = __ldg(Hq + i1), p2 = __ldg(Hq + i2);
                    const float2 h0 = make_float2(0.5f * (p1.x + p2.x) + bias, cj * 0.5f * (p1.y - p2.y));
                    const float2 hw = make_float2(0.5f * (p1.y + p2.y) + bias, -cj * 0.5f * (p1.x - p2.x));
                    const float2 y0 = cmul(x0, h0), yw = cmul(xw, hw);
                    bA[pad16(kz)] = make_float2(s * (y0.x - yw.y), s * (y0.y + yw.x));
                    if (mirror) bB[pad16(kz2)] = make_float2(s * (y0.x + yw.y), s * (yw.x - y0.y));
                }
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

}  // namespace hyena
