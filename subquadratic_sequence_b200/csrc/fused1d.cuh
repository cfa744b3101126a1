// fused1d.cuh -- the single-CTA fused Hyena forward for L <= 16384 and the
// filter-spectrum kernel built from the same FFT passes.
//
// What it computes ("Hyena Hierarchy: Towards Larger Convolutional Language
// Models", abstract: long convolutions interleaved with multiplicative
// gating), per channel-sequence (b, d):
//     z_0 = v,  z_n = x_n * (h_n (*) z_{n-1} + b_n z_{n-1}),  y = z_N,
// with (*) the causal linear convolution over the whole sequence, done by
// the convolution theorem ("Long Context Language Models ... #690", 6:27)
// on a grid zero-padded to P = 2L ("Native Multi-Dimensional Subquadratic
// Operators via Input Dependent Long Convolutions", Handling Boundaries).
// Fusing forward FFT, spectral multiply, inverse FFT and output crop in one
// kernel with the intermediates on chip follows the same page's
// "Implementation: nSubQ / Fused Kernels"; here the gate, the bias and all
// N orders are fused as well, so z never leaves the SM between orders.
//
// Real FFT of P = 2L points as a complex FFT of M = L points: the sequence
// is packed z[m] = u[2m] + i u[2m+1] (m < M/2; the pad half m >= M/2 is
// zero).  With Z = DFT_M(z), w_k = exp(-i pi k / M), Bc = conj(Z[M-k]):
//     U[k]   = ((Z[k] + Bc) - i w_k (Z[k] - Bc)) / 2,  k = 0..M,
// are the P-point spectrum bins.  The bias is folded into the filter
// spectrum: b z = (b delta_0) (*) z, whose DFT is b in every bin, so
// Y[k] = U[k] (H[k] + b).  The inverse is packed the same way:
//     Z'[k] = ((Y[k] + conj Y[M-k]) + i conj(w_k) (Y[k] - conj Y[M-k])) / P
// and z' = IDFT_M(Z') (unnormalised) holds y[2m] + i y[2m+1]; only
// m < M/2 (the first L outputs: the crop) are kept.
//
// The M-point FFT is a Stockham DIT chain of radix-R passes.  Each thread
// keeps E complex values in registers; passes exchange through a padded
// shared buffer.  The first and last pass of every FFT use "folded" thread
// units -- a thread owns column j and column M/R - j -- so that the bins k
// and M - k that the real-FFT split pairs up live in one thread, and the
// forward-last / pair / inverse-first and inverse-last / gate /
// next-forward-first steps never touch shared memory.
#pragma once

#include "hyena_common.cuh"

namespace hyena {

// Radix plan for M = 2^LOG2M: E complex values per thread; boundary radices
// RF (first forward / last inverse pass) and RL (last forward / first
// inverse); up to two middle radices (1 = absent).
template <int LOG2M> struct Plan1d;
#define HYENA_PLAN1D(m, E_, RF_, RM1_, RM2_, RL_)                              \
    template <> struct Plan1d<m> {                                            \
        static constexpr int E = E_, RF = RF_, RM1 = RM1_, RM2 = RM2_, RL = RL_; \
    };
HYENA_PLAN1D(4, 16, 4, 1, 1, 4)
HYENA_PLAN1D(5, 16, 4, 1, 1, 8)
HYENA_PLAN1D(6, 16, 8, 1, 1, 8)
HYENA_PLAN1D(7, 32, 8, 1, 1, 16)
HYENA_PLAN1D(8, 32, 16, 1, 1, 16)
HYENA_PLAN1D(9, 32, 16, 2, 1, 16)
HYENA_PLAN1D(10, 32, 16, 4, 1, 16)
HYENA_PLAN1D(11, 32, 16, 8, 1, 16)
HYENA_PLAN1D(12, 32, 16, 16, 1, 16)
HYENA_PLAN1D(13, 32, 16, 32, 1, 16)
HYENA_PLAN1D(14, 32, 16, 8, 8, 16)
#undef HYENA_PLAN1D

struct Fused1dArgs {
    const void* v;                 // [B][D][L] io
    const void* x[kMaxOrder];      // N pointers, each [B][D][L] io
    void* y;                       // [B][D][L] io
    const float2* H;               // [N][D][L] packed filter spectra ([B][N][D][L] per sample)
    const float* bias;             // [N][D]
    int B, D, N;
    size_t H_bstride;              // slots between samples' spectra (0: shared by the batch)
};

struct Rfft1dArgs {
    const float* h;                // [rows][L]
    float2* H;                     // [rows][L] packed spectra
    int rows;
};

// The real split of one bin pair: the 2M-point spectrum bins X[k] and
// X[M-k] of a real sequence from the M-point transform Z of its packed form
// (Z[k], Z[M-k]); w = exp(-i pi k / M).
__device__ __forceinline__ void split_pair(float2 z1, float2 z2, float2 w, float2& X1, float2& X2)
{
    const float2 bc = cconj(z2);
    const float2 S = cadd(z1, bc);
    const float2 Tw = cmul(w, csub(z1, bc));
    X1 = make_float2(0.5f * (S.x + Tw.y), 0.5f * (S.y - Tw.x));
    X2 = make_float2(0.5f * (S.x - Tw.y), -0.5f * (S.y + Tw.x));
}

// The inverse re-pack of one bin pair (scale s): the M-point inverse
// transform input Z'[k], Z'[M-k] from the spectrum bins Y[k], Y[M-k].
__device__ __forceinline__ void unsplit_pair(float2 y1, float2 y2, float2 w, float s, float2& z1,
                                             float2& z2)
{
    const float2 U = make_float2(y1.x + y2.x, y1.y - y2.y);                 // Y1 + conj Y2
    const float2 V = cmulc(make_float2(y1.x - y2.x, y1.y + y2.y), w);        // conj(w)(Y1 - conj Y2)
    z1 = make_float2(s * (U.x - V.y), s * (U.y + V.x));                     // U + i V
    z2 = make_float2(s * (U.x + V.y), s * (V.x - U.y));                     // conj(U - i V)
}

// Packed spectrum of a real length-L filter zero-padded to 2L: M = L
// complex slots; slot k (1 <= k < L) holds DFT bin k, slot 0 holds
// (bin 0, bin L), both real.  Rows are L * 8 bytes, so 16-byte aligned.

// PAD = true: the causal (linear) convolution; the real sequence of length
// L = M is zero-padded to 2M, so only half the packed inputs are non-zero
// and only half the outputs are kept.  PAD = false: the circular
// convolution of a real sequence of length 2M ("Handling Boundaries":
// circular convolutions for periodic systems), all packed inputs and
// outputs used.
template <int LOG2M, bool PAD = true>
struct Fft1d {
    using P = Plan1d<LOG2M>;
    static constexpr int M = 1 << LOG2M;
    static constexpr int E = P::E;
    static constexpr int T = M / E;                    // threads per sequence
    // sequences per CTA: up to 384 threads, one CTA per SM at 168 registers,
    // so every warp of the SM runs the same pass at the same time and they
    // share the instruction fetch (the unrolled passes are large)
    static constexpr int G = T >= 128 ? (T == 128 ? 3 : 1) : 384 / T;
    static constexpr int THREADS = G * T;
    // exchange buffer, float2; even, so every buffer starts 16-byte aligned
    static constexpr int SMEM_SEQ = (padded_size(M) + 1) & ~1;
    // H_n is staged in its own buffer unless that would not fit next to the
    // exchange buffer; then it goes to the exchange buffer, which is idle
    // between the forward and the inverse FFT, and the staging buffer only
    // holds x_n (at most M/2 float2).
    static constexpr bool H_IN_EXCHANGE = sizeof(float2) * G * (SMEM_SEQ + M) > 227 * 1024;
    static constexpr int STAGE_SEQ = H_IN_EXCHANGE ? M / 2 : M;  // staging buffer, float2
    // packed pairs of real samples per sequence: L/2 = M/2 (causal), M (circular)
    static constexpr int SEQ = PAD ? M / 2 : M;
    static_assert(PAD || !H_IN_EXCHANGE, "circular mode needs the x staging buffer of M pairs");
    static constexpr size_t SMEM_BYTES = sizeof(float2) * G * (SMEM_SEQ + STAGE_SEQ);
    static constexpr size_t SMEM_BYTES_FFT = sizeof(float2) * G * SMEM_SEQ;
    // resident CTAs per SM the register budget is sized for: 168 registers
    // per thread (384 threads per SM) where that allows a CTA at all
    static constexpr int MIN_BLOCKS = THREADS * 168 <= 65536 ? 65536 / (THREADS * 168) : 1;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert((SMEM_SEQ * sizeof(float2)) % 16 == 0 && (STAGE_SEQ * sizeof(float2)) % 16 == 0,
                  "cp.async targets must be 16-byte aligned");
    static_assert(P::RF * P::RM1 * P::RM2 * P::RL == M, "plan");
    static_assert(E % (2 * P::RF) == 0 && E % (2 * P::RL) == 0, "folded units");
    static_assert(M / P::RF >= 2 && M / P::RL >= 2, "folded units");

    // columns of folded unit u for a boundary pass of radix R
    template <int R>
    static __device__ __forceinline__ void unit_cols(int u, int& j0, int& j1)
    {
        constexpr int NCOL = M / R;
        j0 = u;
        j1 = (u == 0) ? NCOL / 2 : NCOL - u;
    }

    // First pass (Ns = 1) from registers in folded layout, radix R.
    template <int R, int SIGN, bool ZERO_HI>
    static __device__ __forceinline__ void pass_first(float2* a, float2* sm, int t)
    {
        static_for<E / (2 * R)>([&](auto cc) {
            constexpr int c = decltype(cc)::value;
            int j[2];
            unit_cols<R>(t + c * T, j[0], j[1]);
            static_for<2>([&](auto hh) {
                constexpr int h = decltype(hh)::value;
                float2* ar = a + (2 * c + h) * R;
                dft<R, SIGN, ZERO_HI>(ar);
                const int pj = pad16(j[h] * R);
                static_for<R>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    // j R + r with R a multiple of 16: pad16(j R) + r + r / 16
                    sm[R % 16 == 0 ? pj + r + r / 16 : pad16(j[h] * R + r)] = ar[r];
                });
            });
        });
        __syncthreads();
    }

    // Exchange layouts.  The first pass writes at a stride of R elements,
    // so its output is padded (element i at pad16(i)).  A middle pass reads
    // and writes 16-element runs that start on a multiple of 16, which are
    // conflict-free in either layout, and writes its output unpadded
    // (element i at i).  The last pass reads the mirrored column NCOL - u of
    // each folded unit: 16 consecutive elements starting one past a multiple
    // of 16, which the padding would split across two 16-element lines (a
    // two-way bank conflict in every half-warp but the first), and which
    // are conflict-free unpadded.  So every pass after a middle pass reads
    // unpadded.
    static constexpr bool HAS_MID = P::RM1 > 1 || P::RM2 > 1;

    // Middle pass: stride NS, radix R, plain column layout j = t + c*T;
    // input padded (PLAIN_IN false) or not, output unpadded.  Column c's
    // twiddle base is chained on column c-1's result so the twiddle
    // arithmetic stays next to the data it multiplies.
    template <int R, int NS, int SIGN, bool PLAIN_IN>
    static __device__ __forceinline__ void pass_mid(float2* a, float2* sm, int t)
    {
        if constexpr (R > 1) {
            static_assert(NS % 16 == 0, "unpadded output: runs of 16 aligned to 16");
            constexpr int C = E / R;
            static_for<C>([&](auto cc) {
                constexpr int c = decltype(cc)::value;
                const int j = t + c * T;
                const int pj = pad16(j);
                static_for<R>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    a[c * R + r] = sm[PLAIN_IN ? j + r * (M / R) : pad16_at<M / R>(j, pj, r)];
                });
            });
            __syncthreads();
            float dep = zero_after(a[0].x);
            static_for<C>([&](auto cc) {
                constexpr int c = decltype(cc)::value;
                const int j = t + c * T;
                const int jm = j % NS;
                float2* ar = a + c * R;
                apply_twiddle_powers<R>(ar, expi_pi<SIGN>(2.0f * (float)jm / (float)(NS * R) + dep));
                dft<R, SIGN>(ar);
                const int base = (j / NS) * NS * R + jm;
                static_for<R>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    sm[base + r * NS] = ar[r];
                });
                dep = zero_after(ar[R - 1].x);
            });
            __syncthreads();
        }
    }

    // Last pass (Ns = M/R) into registers in folded layout; its input is
    // unpadded when a middle pass wrote it.
    template <int R, int SIGN, bool HALF_OUT>
    static __device__ __forceinline__ void pass_last(float2* a, const float2* sm, int t)
    {
        static_for<E / (2 * R)>([&](auto cc) {
            constexpr int c = decltype(cc)::value;
            int j[2];
            unit_cols<R>(t + c * T, j[0], j[1]);
            static_for<2>([&](auto hh) {
                constexpr int h = decltype(hh)::value;
                const int pj = pad16(j[h]);
                static_for<R>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    a[(2 * c + h) * R + r] = sm[HAS_MID ? j[h] + r * (M / R) : pad16_at<M / R>(j[h], pj, r)];
                });
            });
        });
        __syncthreads();
        float dep = zero_after(a[0].x);
        static_for<E / (2 * R)>([&](auto cc) {
            constexpr int c = decltype(cc)::value;
            int j[2];
            unit_cols<R>(t + c * T, j[0], j[1]);
            static_for<2>([&](auto hh) {
                constexpr int h = decltype(hh)::value;
                float2* ar = a + (2 * c + h) * R;
                apply_twiddle_powers<R>(ar, expi_pi<SIGN>(2.0f * (float)j[h] / (float)M + dep));
                dft<R, SIGN, false, HALF_OUT>(ar);
                dep = zero_after(ar[0].x);
            });
        });
    }

    // Forward M-point DFT of the zero-padded packed sequence held in the
    // RF folded layout (elements r < RF/2 of each column); result in the RL
    // folded layout.
    static __device__ __forceinline__ void forward(float2* a, float2* sm, int t)
    {
        pass_first<P::RF, -1, PAD>(a, sm, t);
        pass_mid<P::RM1, P::RF, -1, false>(a, sm, t);
        pass_mid<P::RM2, P::RF * P::RM1, -1, (P::RM1 > 1)>(a, sm, t);
        pass_last<P::RL, -1, false>(a, sm, t);
    }

    // Inverse (unnormalised, sign +1) M-point DFT from the RL folded layout
    // to the RF folded layout, keeping only outputs m < M/2.
    static __device__ __forceinline__ void inverse(float2* a, float2* sm, int t)
    {
        pass_first<P::RL, +1, false>(a, sm, t);
        pass_mid<P::RM2, P::RL, +1, false>(a, sm, t);
        pass_mid<P::RM1, P::RL * P::RM2, +1, (P::RM2 > 1)>(a, sm, t);
        pass_last<P::RF, +1, PAD>(a, sm, t);
    }

    // One pair (k, M-k) of the real-FFT split, the spectral multiply with
    // the bias-folded filter spectrum, and the inverse re-pack.
    //   z1 = Z[k], z2 = Z[M-k]; h1 = H[k], h2 = H[M-k]; w = exp(-i pi k/M)
    // returns Z'[k] in z1 and Z'[M-k] in z2 (scale 1/(2P) included).
    // With G1 = (h1 + b) / (2M), G2 = (h2 + b) / (2M), P = G1 + conj(G2),
    // Q = G1 - conj(G2) and w = c + i s, the split and the re-pack compose
    // to  Z'[k] = (P + s Q) z1 + i c Q conj(z2),
    //     Z'[M-k] = conj(P - s Q) z2 + i c conj(Q) conj(z1).
    static __device__ __forceinline__ void pair(float2& z1, float2& z2, float2 h1, float2 h2,
                                                float2 w, float bias)
    {
        constexpr float sc = 1.0f / (2.0f * (float)M);
        const float bias2 = (2.0f * sc) * bias;
        const float2 P = make_float2(fmaf(sc, h1.x + h2.x, bias2), sc * (h1.y - h2.y));
        const float2 Q = make_float2(sc * (h1.x - h2.x), sc * (h1.y + h2.y));
        const float2 A1 = make_float2(fmaf(w.y, Q.x, P.x), fmaf(w.y, Q.y, P.y));     // P + s Q
        const float2 A2 = make_float2(fmaf(-w.y, Q.x, P.x), fmaf(-w.y, Q.y, P.y));   // P - s Q
        const float2 C = make_float2(w.x * Q.x, w.x * Q.y);                          // c Q
        const float2 a = z1, b = z2;
        z1 = make_float2(fmaf(A1.x, a.x, fmaf(-A1.y, a.y, fmaf(-C.y, b.x, C.x * b.y))),
                         fmaf(A1.x, a.y, fmaf(A1.y, a.x, fmaf(C.x, b.x, C.y * b.y))));
        z2 = make_float2(fmaf(A2.x, b.x, fmaf(A2.y, b.y, fmaf(C.x, a.y, C.y * a.x))),
                         fmaf(A2.x, b.y, fmaf(-A2.y, b.x, fmaf(C.x, a.x, -C.y * a.y))));
    }

    // Spectral step on the RL folded layout for one order; Hs is the
    // packed spectrum row staged in shared memory.  CONJ: multiply by
    // conj(H) + b instead (the adjoint, used by the backward pass).
    template <bool CONJ = false, bool SIGNED = false>
    static __device__ __forceinline__ void spectral(float2* a, const float2* Hs, float bias, int t,
                                                    float him = 1.0f)
    {
        // SIGNED: the imaginary part of H times him (+1: H, -1: conj(H)),
        // chosen at run time
        auto hv = [&](int k) {
            float2 h = Hs[k];
            if (CONJ) h.y = -h.y;
            if (SIGNED) h.y *= him;
            return h;
        };
        constexpr int R = P::RL, NCOL = M / R;
        static_for<E / (2 * R)>([&](auto cc) {
            constexpr int c = decltype(cc)::value;
            const int u = t + c * T;
            float2* a0 = a + (2 * c) * R;
            float2* a1 = a + (2 * c + 1) * R;
            if (u != 0) {
                const int j0 = u;
                float dep = zero_after(a0[0].x);
                const float2 wb = expi_pi<-1>((float)j0 / (float)M + dep);
                static_for<R>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    // the index carries the dependency on the previous pair,
                    // so the spectrum reads are not all hoisted up front
                    const int k = j0 + r * NCOL + __float2int_rz(dep);
                    float2 w = mul_w64<r * 32 / R, -1>(wb);
                    w.x += dep;
                    pair(a0[r], a1[R - 1 - r], hv(k), hv(M - k), w, bias);
                    dep = zero_after(a0[r].x);
                });
            } else {
                // column 0: k = r M/R pairs with M - k = (R - r) M/R; k = 0
                // pairs with the Nyquist bin M (packed in slot 0), k = M/2
                // with itself.
                {
                    const float2 h0 = Hs[0];
                    float2 z1 = a0[0], z2 = a0[0];
                    pair(z1, z2, make_float2(h0.x, 0.0f), make_float2(h0.y, 0.0f),
                         make_float2(1.0f, 0.0f), bias);
                    a0[0] = z1;
                }
                static_for<R / 2 - 1>([&](auto rr) {
                    constexpr int r = decltype(rr)::value + 1;
                    pair(a0[r], a0[R - r], hv(r * NCOL), hv(M - r * NCOL),
                         mul_w64<r * 32 / R, -1>(make_float2(1.0f, 0.0f)), bias);
                });
                {
                    float2 z1 = a0[R / 2], z2 = a0[R / 2];
                    const float2 hm = hv(M / 2);
                    pair(z1, z2, hm, hm, make_float2(0.0f, -1.0f), bias);
                    a0[R / 2] = z1;
                }
                // column NCOL/2: k = M/(2R) + r M/R pairs with register R-1-r
                const float2 wb = expi_pi<-1>(1.0f / (float)(2 * R));
                static_for<R / 2>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    const int k = NCOL / 2 + r * NCOL;
                    pair(a1[r], a1[R - 1 - r], hv(k), hv(M - k), mul_w64<r * 32 / R, -1>(wb), bias);
                });
            }
        });
    }

    // Visit the bin pairs (k, M - k) of the RL folded layout (the real-FFT
    // split): f(i1, i2, k, kind, w) with registers i1 (bin k) and i2 (bin
    // M - k) and w = exp(-i pi k / M); kind 0 = a pair, 1 = bins 0 and M
    // (both in register i1 = i2), 2 = bin M/2 alone (i1 = i2).
    template <typename F>
    static __device__ __forceinline__ void for_each_pair(int t, F&& f)
    {
        constexpr int R = P::RL, NCOL = M / R;
        static_for<E / (2 * R)>([&](auto cc) {
            constexpr int c = decltype(cc)::value;
            const int u = t + c * T;
            if (u != 0) {
                const float2 wb = expi_pi<-1>((float)u / (float)M);
                static_for<R>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    f((2 * c) * R + r, (2 * c + 1) * R + R - 1 - r, u + r * NCOL, 0,
                      mul_w64<r * 32 / R, -1>(wb));
                });
            } else {
                f(0, 0, 0, 1, make_float2(1.0f, 0.0f));
                static_for<R / 2 - 1>([&](auto rr) {
                    constexpr int r = decltype(rr)::value + 1;
                    f(r, R - r, r * NCOL, 0, mul_w64<r * 32 / R, -1>(make_float2(1.0f, 0.0f)));
                });
                f(R / 2, R / 2, M / 2, 2, make_float2(0.0f, -1.0f));
                const float2 wb = expi_pi<-1>(1.0f / (float)(2 * R));
                static_for<R / 2>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    f(R + r, 2 * R - 1 - r, NCOL / 2 + r * NCOL, 0, mul_w64<r * 32 / R, -1>(wb));
                });
            }
        });
    }

    // Visit the data positions m = j + r M/RF (r < RF/2) of the RF folded
    // layout: f(register index, m).
    template <typename F>
    static __device__ __forceinline__ void for_each_io(int t, F&& f)
    {
        constexpr int R = P::RF;
        static_for<E / (2 * R)>([&](auto cc) {
            constexpr int c = decltype(cc)::value;
            int j[2];
            unit_cols<R>(t + c * T, j[0], j[1]);
            static_for<2>([&](auto hh) {
                constexpr int h = decltype(hh)::value;
                static_for<PAD ? R / 2 : R>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    f((2 * c + h) * R + r, j[h] + r * (M / R));
                });
            });
        });
    }
};

// The fused forward: one CTA runs G channel-sequences, all N orders.
// Shared memory per sequence: the padded exchange buffer of the FFT passes
// and a staging buffer that receives H_n (during the forward FFT) and then
// x_n (during the inverse FFT) through asynchronous copies.
// PER_SAMPLE: a spectrum set per sample (input-dependent filters), at
// H + b * H_bstride; otherwise one set shared by the batch.
template <int LOG2M, typename IO, bool PAD = true, bool PER_SAMPLE = false>
__global__ void __launch_bounds__(Fft1d<LOG2M, PAD>::THREADS, Fft1d<LOG2M, PAD>::MIN_BLOCKS)
fused1d_kernel(Fused1dArgs args)
{
    grid_dependency_begin();
    using F = Fft1d<LOG2M, PAD>;
    using IOP = IoPair<IO>;
    using PT = typename IOP::T;
    constexpr int M = F::M, E = F::E, T = F::T;
    constexpr int SEQ = F::SEQ;                          // pairs of samples per sequence
    constexpr int X_BYTES = SEQ * (int)sizeof(PT);       // one sequence of x_n
    extern __shared__ __align__(16) float2 smem_dyn[];

    const int g = threadIdx.x / T, t = threadIdx.x % T;
    const int BD = args.B * args.D;
    const int q_raw = blockIdx.x * F::G + g;
    const bool active = q_raw < BD;
    const int q = active ? q_raw : BD - 1;
    // channel-major order: CTAs next to each other share a filter spectrum
    const int d = q / args.B, b = q % args.B;
    const size_t seq = (size_t)b * args.D + d;
    float2* sm = smem_dyn + g * F::SMEM_SEQ;
    float2* stage = smem_dyn + F::G * F::SMEM_SEQ + g * F::STAGE_SEQ;

    const float2* Hb = PER_SAMPLE ? args.H + (size_t)b * args.H_bstride : args.H;   // this sample's spectra
    // H_0 (or x_1) is in flight while v is loaded and transformed
    if constexpr (!F::H_IN_EXCHANGE)
        cp_async_row(stage, Hb + (size_t)d * M, M * 8, t, T);

    float2 a[E];
    {
        const PT* vp = reinterpret_cast<const PT*>(args.v) + seq * SEQ;
        F::for_each_io(t, [&](int i, int m) { a[i] = IOP::load(vp + m); });
    }
    for (int n = 0; n < args.N; ++n) {
        // select x_n with constant indices (no dynamic indexing of the
        // kernel-parameter array)
        const void* xn = args.x[0];
#pragma unroll
        for (int i = 1; i < kMaxOrder; ++i)
            if (i == n) xn = args.x[i];
        const PT* xg = reinterpret_cast<const PT*>(xn) + seq * SEQ;
        const float2* Hg = Hb + ((size_t)n * args.D + d) * M;
        const float bias = __ldg(args.bias + n * args.D + d);
        const float2* Hs;

        if constexpr (F::H_IN_EXCHANGE) {
            cp_async_row(stage, xg, X_BYTES, t, T);       // x_n during the FFTs
            F::forward(a, sm, t);
            cp_async_row(sm, Hg, M * 8, t, T);            // H_n into the idle exchange buffer
            Hs = sm;
        } else {
            F::forward(a, sm, t);
            Hs = stage;
        }
        cp_async_wait_all();
        __syncthreads();                                  // H_n visible
        F::spectral(a, Hs, bias, t);
        __syncthreads();                                  // H_n consumed
        if constexpr (!F::H_IN_EXCHANGE)
            cp_async_row(stage, xg, X_BYTES, t, T);       // x_n during the inverse FFT
        F::inverse(a, sm, t);
        cp_async_wait_all();
        __syncthreads();                                  // x_n visible
        const PT* xs = reinterpret_cast<const PT*>(stage);
        F::for_each_io(t, [&](int i, int m) {
            const float2 xv = IOP::load_smem(xs + m);
            a[i] = make_float2(a[i].x * xv.x, a[i].y * xv.y);
        });
        __syncthreads();                                  // x_n consumed
        if constexpr (!F::H_IN_EXCHANGE)
            if (n + 1 < args.N)
                cp_async_row(stage, Hb + ((size_t)(n + 1) * args.D + d) * M, M * 8, t, T);
    }
    if (active) {
        PT* yp = reinterpret_cast<PT*>(args.y) + seq * SEQ;
        F::for_each_io(t, [&](int i, int m) { IOP::store(yp + m, a[i]); });
    }
}

// One order of the recurrence per launch, with z in global memory between
// orders: the counterpart of fused1d_kernel that spills z_n to HBM (float32)
// instead of chaining the orders on chip.  It exists to measure what the
// chaining saves ("Native Multi-Dimensional Subquadratic Operators via Input
// Dependent Long Convolutions", Implementation: nSubQ, Memory Efficiency:
// intermediates kept on chip).  z_{n-1} is read as ZIN (v's type for the
// first order, else float), z_n written as ZOUT (y's type for the last
// order, else float); x_n is IO.  zin and zout may be the same buffer: each
// sequence is read whole by the CTA that owns it before that CTA writes it.
struct Fused1dOrderArgs {
    const void* zin;               // [B][D][L] ZIN
    const void* x;                 // [B][D][L] IO (x_n)
    void* zout;                    // [B][D][L] ZOUT
    const float2* H;               // [D][L] packed spectra of order n
    const float* bias;             // [D] (b_n)
    int B, D;
};

template <int LOG2M, typename IO, typename ZIN, typename ZOUT>
__global__ void __launch_bounds__(Fft1d<LOG2M>::THREADS, Fft1d<LOG2M>::MIN_BLOCKS)
fused1d_order_kernel(Fused1dOrderArgs args)
{
    grid_dependency_begin();
    using F = Fft1d<LOG2M>;
    using XP = IoPair<IO>;
    constexpr int M = F::M, E = F::E, T = F::T, SEQ = F::SEQ;
    constexpr int X_BYTES = SEQ * (int)sizeof(typename XP::T);
    extern __shared__ __align__(16) float2 smem_dyn[];

    const int g = threadIdx.x / T, t = threadIdx.x % T;
    const int BD = args.B * args.D;
    const int q_raw = blockIdx.x * F::G + g;
    const bool active = q_raw < BD;
    const int q = active ? q_raw : BD - 1;
    const int d = q / args.B, b = q % args.B;
    const size_t seq = (size_t)b * args.D + d;
    float2* sm = smem_dyn + g * F::SMEM_SEQ;
    float2* stage = smem_dyn + F::G * F::SMEM_SEQ + g * F::STAGE_SEQ;
    const float2* Hg = args.H + (size_t)d * M;
    const typename XP::T* xg = reinterpret_cast<const typename XP::T*>(args.x) + seq * SEQ;
    const float bias = __ldg(args.bias + d);

    if constexpr (!F::H_IN_EXCHANGE) cp_async_row(stage, Hg, M * 8, t, T);
    float2 a[E];
    {
        const typename IoPair<ZIN>::T* zp = reinterpret_cast<const typename IoPair<ZIN>::T*>(args.zin) + seq * SEQ;
        F::for_each_io(t, [&](int i, int m) { a[i] = IoPair<ZIN>::load(zp + m); });
    }
    const float2* Hs;
    if constexpr (F::H_IN_EXCHANGE) {
        cp_async_row(stage, xg, X_BYTES, t, T);
        F::forward(a, sm, t);
        cp_async_row(sm, Hg, M * 8, t, T);
        Hs = sm;
    } else {
        F::forward(a, sm, t);
        Hs = stage;
    }
    cp_async_wait_all();
    __syncthreads();
    F::spectral(a, Hs, bias, t);
    __syncthreads();
    if constexpr (!F::H_IN_EXCHANGE) cp_async_row(stage, xg, X_BYTES, t, T);
    F::inverse(a, sm, t);
    cp_async_wait_all();
    __syncthreads();
    const typename XP::T* xs = reinterpret_cast<const typename XP::T*>(stage);
    F::for_each_io(t, [&](int i, int m) {
        const float2 xv = XP::load_smem(xs + m);
        a[i] = make_float2(a[i].x * xv.x, a[i].y * xv.y);
    });
    if (active) {
        typename IoPair<ZOUT>::T* zp = reinterpret_cast<typename IoPair<ZOUT>::T*>(args.zout) + seq * SEQ;
        F::for_each_io(t, [&](int i, int m) { IoPair<ZOUT>::store(zp + m, a[i]); });
    }
}

// Filter spectra in the packed layout: the DFT of h[row] zero-padded to 2L
// (PAD), or of the unpadded row of length 2M (circular).
template <int LOG2M, bool PAD = true>
__global__ void __launch_bounds__(Fft1d<LOG2M, PAD>::THREADS)
rfft1d_kernel(Rfft1dArgs args)
{
    grid_dependency_begin();
    using F = Fft1d<LOG2M, PAD>;
    constexpr int M = F::M, E = F::E, T = F::T, R = F::P::RL, NCOL = M / R;
    extern __shared__ __align__(16) float2 smem_dyn[];

    const int g = threadIdx.x / T, t = threadIdx.x % T;
    const int row_raw = blockIdx.x * F::G + g;
    const bool active = row_raw < args.rows;
    const size_t row = active ? row_raw : args.rows - 1;
    float2* sm = smem_dyn + g * F::SMEM_SEQ;

    float2 a[E];
    {
        const float2* hp = reinterpret_cast<const float2*>(args.h) + row * F::SEQ;
        F::for_each_io(t, [&](int i, int m) { a[i] = __ldg(hp + m); });
    }
    F::forward(a, sm, t);
    if (!active) return;
    float2* Hrow = args.H + row * M;
    // X[k] = ((Z[k] + Bc) - i w_k (Z[k] - Bc)) / 2,  X[M-k] = conj((.. + ..)) / 2
    auto split = [&](float2 z1, float2 z2, float2 w, int k) {
        const float2 bc = cconj(z2);
        const float2 S = cadd(z1, bc);
        const float2 Tw = cmul(w, csub(z1, bc));
        Hrow[k] = make_float2(0.5f * (S.x + Tw.y), 0.5f * (S.y - Tw.x));
        Hrow[M - k] = make_float2(0.5f * (S.x - Tw.y), -0.5f * (S.y + Tw.x));
    };
    static_for<E / (2 * R)>([&](auto cc) {
        constexpr int c = decltype(cc)::value;
        const int u = t + c * T;
        const float2* a0 = a + (2 * c) * R;
        const float2* a1 = a + (2 * c + 1) * R;
        if (u != 0) {
            const float2 wb = expi_pi<-1>((float)u / (float)M);
            static_for<R>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                split(a0[r], a1[R - 1 - r], mul_w64<r * 32 / R, -1>(wb), u + r * NCOL);
            });
        } else {
            // bins 0 and M are real: packed together in slot 0
            const float2 z = a0[0];
            Hrow[0] = make_float2(z.x + z.y, z.x - z.y);
            static_for<R / 2 - 1>([&](auto rr) {
                constexpr int r = decltype(rr)::value + 1;
                split(a0[r], a0[R - r], mul_w64<r * 32 / R, -1>(make_float2(1.0f, 0.0f)), r * NCOL);
            });
            split(a0[R / 2], a0[R / 2], make_float2(0.0f, -1.0f), M / 2);
            const float2 wb = expi_pi<-1>(1.0f / (float)(2 * R));
            static_for<R / 2>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                split(a1[r], a1[R - 1 - r], mul_w64<r * 32 / R, -1>(wb), NCOL / 2 + r * NCOL);
            });
        }
    });
}

}  // namespace hyena
