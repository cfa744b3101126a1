// fft2d_bwd.cuh -- the backward pass of the 2-D recurrence.
//
// The pages describe the forward only; its gradient follows from the chain
// rule, as in 1-D, with the 2-D linear convolution on the grid padded to
// 2H x 2W ("Native Multi-Dimensional Subquadratic Operators via Input
// Dependent Long Convolutions": Native ND Convolution, Handling
// Boundaries).  With c_n = h_n (*) z_n + b_n z_n, z_{n+1} = x_n c_n and
// g = dL/dz_{n+1} (g = dy for the last order):
//     dx_n  = g c_n,   e = g x_n
//     dh_n += sum_b e (*)' z_n   DFT: E conj(Z_n)            (lags y < H, x < W)
//     db_n  = dh_n[0][0]
//     g    <- h_n (*)' e + b_n e DFT: (conj(H_n) + b_n) E    (outputs y < H, x < W)
// and dv = g after the first order; (*)' is the correlation.
//
// Per wave of images, with the scratch of the forward ([wave][H][W] packed
// row spectra, rows y < H):
//   A. the forward again: rows of v; per order the column step saving the
//      2-D spectrum Z_n of its input, then the inverse rows saving c_n and
//      (but for the last order) gating and transforming z_{n+1};
//   B. per order n = N-1 .. 0: rows: g (dy, or the inverse rows of the
//      scratch), dx_n, e = g x_n, forward rows of e; columns, one CTA per
//      (channel, block of slots) over the channel's images in the wave:
//      forward columns of e, dh spectrum += E conj(Z_n) (a plain
//      read-modify-write: only this CTA touches that block), multiply by
//      (conj(H_n) + b_n) / 2H, inverse columns;
//   then the inverse rows of the scratch give dv.
// After the last wave the accumulated spectra [N][C][2H][W] go through
// inverse columns (rows y < H) and inverse rows: dh_n, and db_n = dh_n[0][0].
// Slot 0 (bins 0 and W of the row transform, packed as one complex
// number) is separated and re-packed through the pair (ky, 2H - ky) as in
// the forward column step.
//
// Per-sample spectra (f.Hs_bstride != 0, input-dependent filters): image
// (b, c) reads sample b's spectra and owns its own dh spectrum (acc
// [B][N][C][2H][W]), so dh is [B][N][C][H][W]; the shared bias's db_n =
// sum_b dh_{b,n}[0][0] is summed by a last small launch.
#pragma once

#include "fft2d.cuh"

namespace hyena {

struct Bwd2dArgs {
    Fft2dArgs f;                   // v, x, Hs, bias, S (scratch), B, C, H, W, q0, nq, n
    const void* dy;                // [B][C][H][W] io
    void* dv;                      // [B][C][H][W] io
    void* dx[kMaxOrder];           // [B][C][H][W] io each
    float2* zsave;                 // [N][wcap][2H][W] spectra of z_n (the wave's images)
    float* csave;                  // [N][wcap][H][W] c_n
    float2* acc;                   // [N][C][2H][W] accumulated dh spectra ([B][N][C][2H][W] per sample)
    float* dh;                     // [N][C][H][W] ([B][N][C][H][W] per sample)
    float* dbias;                  // [N][C]
    int N;                         // order
    int wcap;                      // images a wave holds
    int first;                     // rows MODE 1: g = dy (the last order), else g from the scratch
    int last;                      // rows MODE 0: the last order (c_n saved, no gate, no forward rows)
};

template <typename T>
__device__ __forceinline__ T pick_order(T const* arr, int n)
{
    T p = arr[0];
#pragma unroll
    for (int i = 1; i < kMaxOrder; ++i)
        if (i == n) p = arr[i];
    return p;
}

// Row kernel of the backward.  MODE 0 (A): un-split, inverse rows = c_n,
// saved; but for the last order (ba.last) gate with x_n and forward rows of
// z_{n+1} back into the scratch.  MODE 1 (B): g = dy (ba.first) or
// the inverse rows of the scratch; dx_n = g c_n; e = g x_n; forward rows of
// e.  MODE 2: dv = inverse rows of the scratch.  MODE 3: dh rows from the
// accumulated spectra (rows y < H after the inverse columns), db = dh[0][0].
// 3-D volumes (f.zp != 0) are Z planes of Hp rows: f.H = Z Hp rows a volume.
template <int LOG2W, typename IO, int MODE, bool PAD = true>
__global__ void __launch_bounds__(Fft1d<LOG2W, PAD>::THREADS)
fft2d_bwd_row_kernel(Bwd2dArgs ba)
{
    grid_dependency_begin();
    const Fft2dArgs& a = ba.f;
    using R = Fft2dRows<LOG2W, PAD>;
    using F = typename R::F;
    using IOP = IoPair<IO>;
    using PT = typename IOP::T;
    constexpr int W = R::W, E = F::E, T = F::T, SEQ = F::SEQ;
    extern __shared__ __align__(16) float2 smem_rb[];

    const int g = threadIdx.x / T, t = threadIdx.x % T;
    const int rows = a.nq * a.H;
    const int qr_raw = blockIdx.x * F::G + g;
    const bool active = qr_raw < rows;
    const int qr = active ? qr_raw : rows - 1;
    const int qi = qr / a.H, yrow = qr % a.H;
    const int q = a.q0 + qi;
    float2* sm = smem_rb + g * F::SMEM_SEQ;
    float2 arr[E];

    if constexpr (MODE == 3) {
        // q: filter row n*C + c of the accumulated spectra [2H][W] (3-D:
        // row y of plane z of [2Z][2H][W], yrow = z Hp + y)
        constexpr int RP = PAD ? 2 : 1;
        const float2* row;
        if (a.zp == 0) {
            row = ba.acc + ((size_t)q * RP * a.H + yrow) * W;
        } else {
            const int z = yrow / a.Hp, y = yrow - z * a.Hp;
            row = ba.acc + (((size_t)q * RP * a.zp + z) * RP * a.Hp + y) * W;
        }
        R::unsplit_inverse(arr, sm, row, t);
        if (active) {
            float2* dhp = reinterpret_cast<float2*>(ba.dh + ((size_t)q * a.H + yrow) * 2 * SEQ);
            F::for_each_io(t, [&](int i, int m) {
                dhp[m] = arr[i];
                if (yrow == 0 && m == 0 && a.Hs_bstride == 0) ba.dbias[q] = arr[i].x;   // db_n = dh_n[0][0]
            });
        }
        return;
    } else {
        const int c = q / a.B, b = q % a.B;
        const size_t img = (size_t)b * a.C + c;
        const size_t off = (img * a.H + yrow) * SEQ;             // value pairs of this grid row
        float2* row = scratch_row<PAD>(a, qi, yrow);
        float2* cs = reinterpret_cast<float2*>(ba.csave) + (((size_t)a.n * ba.wcap + qi) * a.H + yrow) * SEQ;
        const PT* xp = reinterpret_cast<const PT*>(pick_order(a.x, a.n)) + off;
        if constexpr (MODE == 0) {
            R::unsplit_inverse(arr, sm, row, t);                  // c_n
            if (active) F::for_each_io(t, [&](int i, int m) { cs[m] = arr[i]; });
            if (!ba.last) {
                F::for_each_io(t, [&](int i, int m) {
                    const float2 xv = IOP::load(xp + m);
                    arr[i] = make_float2(arr[i].x * xv.x, arr[i].y * xv.y);
                });
                R::forward_split(arr, sm, row, t, active);
            }
        } else if constexpr (MODE == 1) {
            if (ba.first) {
                const PT* gp = reinterpret_cast<const PT*>(ba.dy) + off;
                F::for_each_io(t, [&](int i, int m) { arr[i] = IOP::load(gp + m); });
            } else {
                R::unsplit_inverse(arr, sm, row, t);              // g = dL/dz_{n+1}
            }
            PT* dxp = reinterpret_cast<PT*>(pick_order(ba.dx, a.n)) + off;
            // all loads first, then the stores: one latency, not one per value
            constexpr int RF = F::P::RF;
            constexpr int NIO = PAD ? E / 2 : E;                     // io registers
            auto io_slot = [](int i) { return PAD ? (i / RF) * (RF / 2) + i % RF : i; };   // -> [0, NIO)
            float2 cv[NIO], xv[NIO];
            F::for_each_io(t, [&](int i, int m) {
                cv[io_slot(i)] = cs[m];
                xv[io_slot(i)] = IOP::load(xp + m);
            });
            F::for_each_io(t, [&](int i, int m) {
                const float2 c_ = cv[io_slot(i)], x_ = xv[io_slot(i)];
                if (active) IOP::store(dxp + m, make_float2(arr[i].x * c_.x, arr[i].y * c_.y));
                arr[i] = make_float2(arr[i].x * x_.x, arr[i].y * x_.y);      // e
            });
            R::forward_split(arr, sm, row, t, active);
        } else {
            R::unsplit_inverse(arr, sm, row, t);                  // dv = dL/dz_0
            if (active) {
                PT* dvp = reinterpret_cast<PT*>(ba.dv) + off;
                F::for_each_io(t, [&](int i, int m) { IOP::store(dvp + m, arr[i]); });
            }
        }
    }
}

// Column kernel of the backward (2H-point columns, TC slots a CTA).
// MODE 0 (A): per image, forward columns of rows y < H, the spectrum saved
// to zsave[n], multiply by (H_n + b_n) / 2H, inverse columns, rows y < H
// back.  MODE 1 (B): per (channel, block of slots), over the channel's
// images in the wave: forward columns of e, acc += E conj(Z_n), multiply
// by (conj(H_n) + b_n) / 2H, inverse columns, rows y < H back.  MODE 2:
// inverse columns of the accumulated spectra (all 2H rows), scaled by
// 1/2H, rows y < H back in place.
template <int LOG2H2, int MODE, bool PAD = true>
__global__ void __launch_bounds__(Fft2dCols<LOG2H2, PAD>::THREADS, Fft2dCols<LOG2H2, PAD>::MIN_BLOCKS)
fft2d_bwd_col_kernel(Bwd2dArgs ba)
{
    grid_dependency_begin();
    const Fft2dArgs& a = ba.f;
    using CL = Fft2dCols<LOG2H2, PAD>;
    using FC = typename CL::FC;
    constexpr int H2 = CL::H2, TC = CL::TC, HH = H2 / 2, V = FC::V;
    constexpr int ROWS = PAD ? HH : H2;                 // grid rows in a column
    constexpr int VL = PAD ? V / 2 : V;                 // registers holding grid rows
    constexpr float s = 1.0f / (float)H2;
    const int W = a.W;
    const int CTAS_PER_ROW = W / TC;
    extern __shared__ __align__(16) float2 smem_cb[];
    const int tid = threadIdx.x;
    const int cc = tid % TC, t = tid / TC;
    const int kx = (blockIdx.x % CTAS_PER_ROW) * TC + cc;
    const int unit = blockIdx.x / CTAS_PER_ROW;               // image (A), channel (B) or filter row (2)
    float2* buf = smem_cb + cc * CL::STRIDE;
    const int pt = pad16(t);
    float2 reg[V];

    if constexpr (MODE == 2) {
        float2* col = ba.acc + (size_t)unit * H2 * W + kx;
        static_for<V>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            buf[pad16_at<H2 / V>(t, pt, r)] = col[(size_t)(t + r * (H2 / V)) * W];
        });
        __syncthreads();
        FC::template run<+1, true>(buf, reg, t);
        static_for<VL>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            col[(size_t)(t + r * (H2 / V)) * W] = make_float2(reg[r].x * s, reg[r].y * s);
        });
        return;
    } else {
        // images this CTA takes: one (A), or the wave's images of one channel (B)
        int qa, qb, c;
        if constexpr (MODE == 0) {
            qa = a.q0 + unit;
            qb = qa + 1;
            c = qa / a.B;
        } else {
            c = a.q0 / a.B + unit;
            qa = max(a.q0, c * a.B);
            qb = min(a.q0 + a.nq, (c + 1) * a.B);
        }
        const float bias = __ldg(a.bias + a.n * a.C + c);
        const bool ps = a.Hs_bstride != 0;
        for (int q = qa; q < qb; ++q) {
            const int qi = q - a.q0;
            // per-sample spectra: sample b's filters and its own dh spectrum
            const size_t sb = ps ? (size_t)(q % a.B) : 0;
            const float2* Hc = a.Hs + sb * a.Hs_bstride + ((size_t)a.n * a.C + c) * H2 * W + kx;
            float2* accc = ba.acc + ((sb * ba.N + a.n) * a.C + c) * H2 * W + kx;
            float2* col = a.S + (size_t)qi * ROWS * W + kx;
            float2* zc = ba.zsave + ((size_t)a.n * ba.wcap + qi) * H2 * W + kx;
            static_for<VL>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                buf[pad16_at<H2 / V>(t, pt, r)] = col[(size_t)(t + r * (H2 / V)) * W];
            });
            __syncthreads();
            FC::template run<-1, true, PAD>(buf, reg, t);
            if constexpr (MODE == 0)
                static_for<V>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    zc[(size_t)(t + r * (H2 / V)) * W] = reg[r];
                });
            static_for<V>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                buf[pad16_at<H2 / V>(t, pt, r)] = reg[r];
            });
            __syncthreads();
            // the forward multiplies by H + b; the backward by conj(H) + b
            constexpr float cj = MODE == 0 ? 1.0f : -1.0f;
            // (runtime loops over the thread's rows: fully unrolled, the
            // compiler hoists every load and runs out of registers)
            if (kx != 0) {
                // K rows at a time, every load of the group before its stores:
                // interleaved, each accumulator load would wait for the store
                // before it
                constexpr int K = 4;
                static_assert(V % K == 0, "row groups");
#pragma unroll 1
                for (int r0 = 0; r0 < V; r0 += K) {
                    float2 ev[K], hv[K], zv[K], av[K];
                    static_for<K>([&](auto jj) {
                        constexpr int j = decltype(jj)::value;
                        const int ky = t + (r0 + j) * (H2 / V);
                        ev[j] = buf[pad16(ky)];
                        hv[j] = __ldg(Hc + (size_t)ky * W);
                        if constexpr (MODE == 1) {
                            zv[j] = zc[(size_t)ky * W];
                            av[j] = accc[(size_t)ky * W];
                        }
                    });
                    static_for<K>([&](auto jj) {
                        constexpr int j = decltype(jj)::value;
                        const int ky = t + (r0 + j) * (H2 / V);
                        if constexpr (MODE == 1) accc[(size_t)ky * W] = cadd(av[j], cmulc(ev[j], zv[j]));
                        buf[pad16(ky)] = cmul(ev[j], make_float2((hv[j].x + bias) * s, cj * hv[j].y * s));
                    });
                }
            } else {
                // slot 0 = (bin-0 column) + i (bin-W column): separate both
                // through the pair (ky, 2H - ky), take each product, re-pack
#pragma unroll 1
                for (int r = 0; r < V; ++r) {
                    const int ky = t + r * (H2 / V);
                    if (ky > HH) continue;
                    const int kn = (H2 - ky) % H2;
                    const float2 c1 = buf[pad16(ky)], c2 = buf[pad16(kn)];
                    // X0 = (C1 + conj C2)/2,  XW = (C1 - conj C2)/(2i)
                    const float2 x0 = make_float2(0.5f * (c1.x + c2.x), 0.5f * (c1.y - c2.y));
                    const float2 xw = make_float2(0.5f * (c1.y + c2.y), -0.5f * (c1.x - c2.x));
                    if constexpr (MODE == 1) {
                        const float2 z1 = zc[(size_t)ky * W], z2 = zc[(size_t)kn * W];
                        const float2 z0 = make_float2(0.5f * (z1.x + z2.x), 0.5f * (z1.y - z2.y));
                        const float2 zw = make_float2(0.5f * (z1.y + z2.y), -0.5f * (z1.x - z2.x));
                        const float2 p0 = cmulc(x0, z0), pw = cmulc(xw, zw);
                        // bin ky: P0 + i PW; bin 2H - ky: conj(P0) + i conj(PW)
                        accc[(size_t)ky * W] = cadd(accc[(size_t)ky * W], make_float2(p0.x - pw.y, p0.y + pw.x));
                        if (kn != ky)
                            accc[(size_t)kn * W] = cadd(accc[(size_t)kn * W], make_float2(p0.x + pw.y, pw.x - p0.y));
                    }
                    const float2 p1 = __ldg(Hc + (size_t)ky * W), p2 = __ldg(Hc + (size_t)kn * W);
                    const float2 h0 = make_float2(0.5f * (p1.x + p2.x) + bias, cj * 0.5f * (p1.y - p2.y));
                    const float2 hw = make_float2(0.5f * (p1.y + p2.y) + bias, -cj * 0.5f * (p1.x - p2.x));
                    const float2 y0 = cmul(x0, h0), yw = cmul(xw, hw);
                    buf[pad16(ky)] = make_float2(s * (y0.x - yw.y), s * (y0.y + yw.x));
                    if (kn != ky) buf[pad16(kn)] = make_float2(s * (y0.x + yw.y), s * (yw.x - y0.y));
                }
            }
            __syncthreads();
            FC::template run<+1, true>(buf, reg, t);
            static_for<VL>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                col[(size_t)(t + r * (H2 / V)) * W] = reg[r];
            });
        }
    }
}

// Per-sample spectra: db_n[c] = sum_b dh_{b,n}[c][0][0], one thread per
// (n, c), the samples in order (deterministic).  A grid of f.H rows holds
// f.W reals a row (PAD: one real per slot) or 2 f.W (circular: two).
template <bool PAD>
__global__ void __launch_bounds__(256) db2d_sum_kernel(Bwd2dArgs ba)
{
    grid_dependency_begin();
    const int rows = ba.N * ba.f.C;
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const size_t plane = (size_t)ba.f.H * (PAD ? 1 : 2) * ba.f.W;
    float s = 0.0f;
    for (int b = 0; b < ba.f.B; ++b) s += ba.dh[((size_t)b * rows + r) * plane];
    ba.dbias[r] = s;
}

}  // namespace hyena
