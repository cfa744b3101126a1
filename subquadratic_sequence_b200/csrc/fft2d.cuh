// fft2d.cuh -- the 2-D Hyena forward and 2-D filter spectra.
//
// Per image (b, c) and order n: the linear 2-D convolution of z_{n-1}
// [H][W] with the filter h_n [H][W] (offsets 0..H-1 x 0..W-1) through the
// 2-D DFT of the grid zero-padded to 2H x 2W ("Native Multi-Dimensional
// Subquadratic Operators via Input Dependent Long Convolutions": Native ND
// Convolution, Handling Boundaries), plus the bias, cropped to [0,H) x
// [0,W) and gated by x_n -- the same recurrence as the 1-D operator.
//
// Real 2-D DFT, packed:
//  * rows: each real row of 2W samples (only x < W non-zero) is the packed
//    W-point complex sequence u[2m] + i u[2m+1]; its W-point FFT and the
//    real split give row bins 0..W.  Bins 0 and W are real and share slot
//    0 as (bin 0, bin W), so a row spectrum is exactly W complex slots.
//  * columns: each slot column (2H points, rows y >= H zero) is transformed
//    by a 2H-point complex FFT.  Slot 0 then holds the transform of the
//    complex column (bin-0 column) + i (bin-W column): both are transforms
//    of real sequences, separated through the pair (ky, 2H - ky).
// The 2-D spectrum of a filter is therefore [2H][W] complex in this packed
// form.  The spectral step multiplies every bin by (H + b) / (2H) and the
// row un-split carries the remaining 1 / (2W) of the inverse.
//
// One order is a column launch (column FFTs, spectral multiply, inverse
// column FFTs, keep rows y < H) and a row launch (row un-split, inverse
// row FFTs, crop x < W, gate, and -- unless this was the last order -- the
// next order's forward row FFTs and split).  The first order starts with a
// row launch that reads v.  Images go in waves whose scratch ([H][W]
// complex per image) stays in L2.
#pragma once

#include "fourstep.cuh"
#include "fused1d.cuh"

namespace hyena {

struct Fft2dArgs {
    const void* v;                 // [B][C][H][W] io
    const void* x[kMaxOrder];      // x_1..x_N, [B][C][H][W] io
    void* y;                       // [B][C][H][W] io
    const float2* Hs;              // [N][C][2H][W] packed 2-D spectra (column kernel)
    const float* bias;             // [N][C]
    float2* S;                     // scratch [wave][H][W] complex (conv) / spectra (filters)
    int B, C, H;
    int W;                         // slots per row: the grid width (padded), half of it (circular)
    int q0;                        // first image of the wave (channel-major index)
    int nq;                        // images in the wave
    int n;                         // order handled by this launch
    size_t Hs_bstride;             // slots between samples' spectra (0: shared by the batch)
    // 3-D volumes [Z][Hp][W] as Z planes per image (0 for 2-D grids): the
    // row kernel then sees H = Z * Hp rows per image and keeps every plane
    // at a pitch of 2 Hp rows in the scratch (and of 2 Z planes per filter
    // in the spectra)
    int zp, Hp;
};

// Scratch row of row index yrow of image qi (2-D: [H][W] per image; 3-D:
// plane z = yrow / Hp at a pitch of 2 Hp rows, or Hp rows when circular).
template <bool PAD>
__device__ __forceinline__ float2* scratch_row(const Fft2dArgs& a, int qi, int yrow)
{
    if (a.zp == 0) return a.S + ((size_t)qi * a.H + yrow) * a.W;
    const int z = yrow / a.Hp, y = yrow - z * a.Hp;
    return a.S + (((size_t)qi * a.zp + z) * (PAD ? 2 : 1) * a.Hp + y) * a.W;
}

// Rows as packed real transforms of 2M points: a row of W = M values
// zero-padded to 2W (PAD), or of W = 2M values taken whole (circular); M
// slots per row, slot 0 holding bins 0 and M.
template <int LOG2M, bool PAD = true>
struct Fft2dRows {
    using F = Fft1d<LOG2M, PAD>;
    static constexpr int W = 1 << LOG2M;               // slots per row

    // forward row FFT of the registers (every thread: the passes hold
    // barriers) and, if `store`, the split into a packed row
    static __device__ __forceinline__ void forward_split(float2* a, float2* sm, float2* row, int t,
                                                         bool store)
    {
        F::forward(a, sm, t);
        if (!store) return;
        F::for_each_pair(t, [&](int i1, int i2, int k, int kind, float2 w) {
            if (kind == 1) {
                const float2 z = a[i1];
                row[0] = make_float2(z.x + z.y, z.x - z.y);          // bins 0 and W
            } else {
                float2 X1, X2;
                split_pair(a[i1], a[i2], w, X1, X2);
                row[k] = X1;
                if (kind == 0) row[W - k] = X2;
            }
        });
    }

    // load a packed row into the registers as the inverse FFT's input
    // (scale 1/(2W)) and run the inverse row FFT (outputs x < W kept)
    static __device__ __forceinline__ void unsplit_inverse(float2* a, float2* sm, const float2* row, int t)
    {
        constexpr float s = 1.0f / (2.0f * (float)W);
        F::for_each_pair(t, [&](int i1, int i2, int k, int kind, float2 w) {
            float2 z1, z2;
            if (kind == 1) {
                const float2 p = row[0];
                unsplit_pair(make_float2(p.x, 0.0f), make_float2(p.y, 0.0f), w, s, z1, z2);
                a[i1] = z1;
            } else if (kind == 2) {
                const float2 yk = row[k];
                unsplit_pair(yk, yk, w, s, z1, z2);
                a[i1] = z1;
            } else {
                unsplit_pair(row[k], row[W - k], w, s, z1, z2);
                a[i1] = z1;
                a[i2] = z2;
            }
        });
        F::inverse(a, sm, t);
    }
};

// Row kernel.  MODE 0: forward rows from v into the scratch; 1: un-split,
// inverse rows, gate, forward rows back into the scratch; 2: un-split,
// inverse rows, gate, store y; 3: forward rows of the filters h into rows
// y < H of the packed spectra (S = spectra, C = filter rows).  PAD: rows
// zero-padded to twice their width, else circular.
template <int LOG2M, typename IO, int MODE, bool PAD = true>
__global__ void __launch_bounds__(Fft1d<LOG2M, PAD>::THREADS)
fft2d_row_kernel(Fft2dArgs a)
{
    grid_dependency_begin();
    using R = Fft2dRows<LOG2M, PAD>;
    using F = typename R::F;
    using IOP = IoPair<IO>;
    using PT = typename IOP::T;
    constexpr int W = R::W, E = F::E, T = F::T, SEQ = F::SEQ;   // slots, -, -, value pairs per row
    constexpr int RP = PAD ? 2 : 1;                              // spectrum rows (planes) per grid row (plane)
    extern __shared__ __align__(16) float2 smem_r2[];

    const int g = threadIdx.x / T, t = threadIdx.x % T;
    const int rows = a.nq * a.H;
    const int qr_raw = blockIdx.x * F::G + g;
    const bool active = qr_raw < rows;
    const int qr = active ? qr_raw : rows - 1;
    const int qi = qr / a.H, yrow = qr % a.H;
    const int q = a.q0 + qi;
    float2* sm = smem_r2 + g * F::SMEM_SEQ;
    float2 arr[E];

    if constexpr (MODE == 0 || MODE == 3) {
        size_t img;
        float2* row;
        if constexpr (MODE == 0) {
            const int c = q / a.B, b = q % a.B;
            img = (size_t)b * a.C + c;
            row = scratch_row<PAD>(a, qi, yrow);
        } else {
            img = (size_t)q;                                  // filter row n*C + c
            if (a.zp == 0) {
                row = a.S + ((size_t)q * RP * a.H + yrow) * W;
            } else {                                          // plane z of [RP Z][RP Hp][W]
                const int z = yrow / a.Hp, y = yrow - z * a.Hp;
                row = a.S + (((size_t)q * RP * a.zp + z) * RP * a.Hp + y) * W;
            }
        }
        const PT* vp = reinterpret_cast<const PT*>(a.v) + (img * a.H + yrow) * SEQ;
        F::for_each_io(t, [&](int i, int m) { arr[i] = IOP::load(vp + m); });
        R::forward_split(arr, sm, row, t, active);
    } else {
        const int c = q / a.B, b = q % a.B;
        const size_t img = (size_t)b * a.C + c;
        float2* row = scratch_row<PAD>(a, qi, yrow);
        R::unsplit_inverse(arr, sm, row, t);
        const void* xn = a.x[0];
#pragma unroll
        for (int i = 1; i < kMaxOrder; ++i)
            if (i == a.n) xn = a.x[i];
        const size_t off = (img * a.H + yrow) * SEQ;
        const PT* xp = reinterpret_cast<const PT*>(xn) + off;
        F::for_each_io(t, [&](int i, int m) {
            const float2 xv = IOP::load(xp + m);
            arr[i] = make_float2(arr[i].x * xv.x, arr[i].y * xv.y);
        });
        if constexpr (MODE == 2) {
            if (active) {
                PT* yp = reinterpret_cast<PT*>(a.y) + off;
                F::for_each_io(t, [&](int i, int m) { IOP::store(yp + m, arr[i]); });
            }
        } else {
            R::forward_split(arr, sm, row, t, active);
        }
    }
}

template <int LOG2H2, bool PAD = true>
struct Fft2dCols {
    using FC = SmemFft<LOG2H2>;
    static constexpr int H2 = 1 << LOG2H2;             // 2H
    // TC columns per CTA (column index fastest across threads: every global
    // access is a TC-element run); about 256 threads
    static constexpr int TC = (256 / FC::T) > 16 ? 16 : ((256 / FC::T) < 4 ? 4 : 256 / FC::T);
    static constexpr int THREADS = TC * FC::T;
    static constexpr int STRIDE = stride_mod16(H2, 16 / TC);
    static constexpr size_t SMEM = sizeof(float2) * TC * STRIDE;
    // resident CTAs per SM: up to three, as shared memory allows and with at
    // least 80 registers per thread (120 with 32 values per thread); more
    // for circular columns, whose whole column is live in registers
    static constexpr int REGS = PAD ? (FC::V == 32 ? 120 : 80) : (FC::V == 32 ? 160 : 104);
    static constexpr int BY_SMEM = 3 * SMEM <= 227 * 1024 ? 3 : (2 * SMEM <= 227 * 1024 ? 2 : 1);
    static constexpr int BY_REGS = 65536 / (THREADS * REGS) < 1 ? 1 : 65536 / (THREADS * REGS);
    static constexpr int MIN_BLOCKS = BY_SMEM < BY_REGS ? BY_SMEM : BY_REGS;
    static_assert(THREADS <= 1024 && SMEM <= 227 * 1024, "column kernel geometry");
};

// Column kernel, columns of H2 = 2H points (PAD: rows y < H, zero-padded)
// or H2 = H points (circular).  MODE 0: column FFTs of the scratch,
// spectral multiply with the packed 2-D filter spectrum and the bias,
// inverse column FFTs, rows y < H back to the scratch.  MODE 1: forward
// column FFTs of each plane (the packed spectra, or 3-D scratch planes),
// all H2 rows written back.  MODE 2 (3-D): inverse column FFTs of all H2
// rows of each plane, rows y < H written back.  In both, with zp and PAD,
// plane q is plane q % zp of spectrum q / zp at a pitch of 2 zp planes
// (the filter spectra, the backward's accumulated spectra).
template <int LOG2H2, int MODE, bool PAD = true>
__global__ void __launch_bounds__(Fft2dCols<LOG2H2, PAD>::THREADS, Fft2dCols<LOG2H2, PAD>::MIN_BLOCKS)
fft2d_col_kernel(Fft2dArgs a)
{
    constexpr bool SPECTRUM = MODE == 1;
    grid_dependency_begin();
    using CL = Fft2dCols<LOG2H2, PAD>;
    using FC = typename CL::FC;
    constexpr int H2 = CL::H2, TC = CL::TC, HH = H2 / 2, V = FC::V;
    constexpr int ROWS = PAD ? HH : H2;                 // grid rows in a column
    constexpr int VL = PAD ? V / 2 : V;                 // registers holding grid rows
    const int W = a.W;
    const int CTAS_PER_IMG = W / TC;
    extern __shared__ __align__(16) float2 smem_c2[];

    const int qi = blockIdx.x / CTAS_PER_IMG;
    const int kx0 = (blockIdx.x % CTAS_PER_IMG) * TC;
    const int q = a.q0 + qi;
    const int tid = threadIdx.x;
    const int cc = tid % TC, t = tid / TC;
    const int kx = kx0 + cc;
    float2* buf = smem_c2 + cc * CL::STRIDE;
    // rows of this image's column kx: scratch [H][W] or planes [2H][W]
    const size_t pq = (MODE != 0 && a.zp && PAD) ? (size_t)(q / a.zp) * 2 * a.zp + q % a.zp : (size_t)q;
    float2* col = MODE != 0 ? a.S + pq * H2 * W + kx : a.S + (size_t)qi * ROWS * W + kx;
    float2 reg[V];
    const int pt = pad16(t);

    if constexpr (MODE == 2) {
        // inverse column FFT of all H2 rows, grid rows back
        static_for<V>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            buf[pad16_at<H2 / V>(t, pt, r)] = col[(size_t)(t + r * (H2 / V)) * W];
        });
        __syncthreads();
        FC::template run<+1, true>(buf, reg, t);
        static_for<VL>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            col[(size_t)(t + r * (H2 / V)) * W] = reg[r];
        });
        return;
    }
    static_for<VL>([&](auto rr) {
        constexpr int r = decltype(rr)::value;
        buf[pad16_at<H2 / V>(t, pt, r)] = col[(size_t)(t + r * (H2 / V)) * W];
    });
    __syncthreads();
    FC::template run<-1, true, PAD>(buf, reg, t);
    if constexpr (SPECTRUM) {
        static_for<V>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            col[(size_t)(t + r * (H2 / V)) * W] = reg[r];
        });
        return;
    } else {
        static_for<V>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            buf[pad16_at<H2 / V>(t, pt, r)] = reg[r];
        });
        __syncthreads();
        // spectral multiply by (H + b) / H2
        const int c = q / a.B;
        const float bias = __ldg(a.bias + a.n * a.C + c);
        const float2* Hc = a.Hs + (size_t)(q % a.B) * a.Hs_bstride + ((size_t)a.n * a.C + c) * H2 * W + kx;
        constexpr float s = 1.0f / (float)H2;
        if (kx != 0) {
            static_for<V>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                const int ky = t + r * (H2 / V);
                const float2 hv = __ldg(Hc + (size_t)ky * W);
                const int pk = pad16_at<H2 / V>(t, pt, r);
                buf[pk] = cmul(buf[pk], make_float2((hv.x + bias) * s, hv.y * s));
            });
        } else {
            // slot 0 = (bin-0 column) + i (bin-W column): separate both
            // through the pair (ky, 2H - ky), multiply each by its own
            // filter column, and re-pack
            static_for<V>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                const int ky = t + r * (H2 / V);
                if (ky <= HH) {
                    const int kn = (H2 - ky) % H2;
                    const float2 c1 = buf[pad16(ky)], c2 = buf[pad16(kn)];
                    const float2 p1 = __ldg(Hc + (size_t)ky * W), p2 = __ldg(Hc + (size_t)kn * W);
                    // X0 = (C1 + conj C2)/2,  XW = (C1 - conj C2)/(2i); same for the filter
                    const float2 x0 = make_float2(0.5f * (c1.x + c2.x), 0.5f * (c1.y - c2.y));
                    const float2 xw = make_float2(0.5f * (c1.y + c2.y), -0.5f * (c1.x - c2.x));
                    const float2 h0 = make_float2(0.5f * (p1.x + p2.x) + bias, 0.5f * (p1.y - p2.y));
                    const float2 hw = make_float2(0.5f * (p1.y + p2.y) + bias, -0.5f * (p1.x - p2.x));
                    const float2 y0 = cmul(x0, h0), yw = cmul(xw, hw);
                    // bin ky: Y0 + i YW; bin 2H - ky: conj(Y0) + i conj(YW)
                    buf[pad16(ky)] = make_float2(s * (y0.x - yw.y), s * (y0.y + yw.x));
                    if (kn != ky)
                        buf[pad16(kn)] = make_float2(s * (y0.x + yw.y), s * (yw.x - y0.y));
                }
            });
        }
        __syncthreads();
        FC::template run<+1, true>(buf, reg, t);
        static_for<VL>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            col[(size_t)(t + r * (H2 / V)) * W] = reg[r];
        });
    }
}

}  // namespace hyena
