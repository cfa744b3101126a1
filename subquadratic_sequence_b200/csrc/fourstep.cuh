// fourstep.cuh -- the Hyena forward for sequences too long for one SM
// (L > 16384), and the filter spectra at those lengths.
//
// Same operator and same real-FFT packing as fused1d.cuh: the 2L-point real
// FFT of the zero-padded sequence is an M = L point complex FFT of
// z[m] = u[2m] + i u[2m+1].  Here that FFT is split four-step, M = M1 * M2:
//   n = n2 + M2 n1,  k = k1 + M1 k2,
//   Z[k1 + M1 k2] = sum_n2 W_M2^{n2 k2} W_M^{n2 k1} sum_n1 z[n2 + M2 n1] W_M1^{n1 k1}
// and its inverse the same way backwards.  One order of the recurrence is
// two launches:
//   row kernel    per pair of rows (k1, M1 - k1): the M2-point row FFTs,
//                 the real split + bias-folded spectral multiply + inverse
//                 re-pack (bin k pairs with bin M - k, which sits in row
//                 M1 - k1), the inverse row FFTs and their twiddle;
//   column kernel per block of columns n2: the inverse M1-point column
//                 FFTs, the crop (n1 < M1/2 is the first L outputs), the
//                 gate by x_n, and -- unless this was the last order -- the
//                 next order's forward column FFTs and twiddle.
// The first order starts with a column kernel that reads v.  The scratch
// (one M-point complex array per sequence) is read and written in place;
// sequences go through in waves small enough for the wave's scratch to stay
// resident in L2.
#pragma once

#include "hyena_common.cuh"

namespace hyena {

__host__ __device__ constexpr int ipow16(int p) { return p <= 0 ? 1 : 16 * ipow16(p - 1); }

// Shared-memory buffer stride (float2) that is >= padded_size(n) and
// congruent to `mod16` modulo 16: neighbouring buffers then start on
// different banks.
__host__ __device__ constexpr int stride_mod16(int n, int mod16)
{
    const int p = padded_size(n);
    return p + ((mod16 - p % 16) + 16) % 16;
}

// One S = 2^LOG2S point FFT held in a padded shared buffer and transformed
// by T = S/V threads (V values each), Stockham DIT, natural order in and
// out.  V = 32 for S = 512 and 1024 (two passes: radix S/32, then 32),
// else 16 (passes of radix 16 after a first pass of S / 16^(NP-1)).  Several
// transforms run side by side in a CTA; every pass ends in a
// __syncthreads() of the whole CTA.  On return a[r] holds X[t + r S/V].
template <int LOG2S>
struct SmemFft {
    static_assert(LOG2S >= 4, "S >= 16");
    static constexpr int S = 1 << LOG2S;
    static constexpr int V = (LOG2S == 9 || LOG2S == 10) ? 32 : 16;          // values per thread
    static constexpr int T = S / V;
    static constexpr int NP = V == 32 ? 2 : (LOG2S + 3) / 4;                 // passes
    static constexpr int R0 = V == 32 ? S / 32
                            : (LOG2S % 4 == 0) ? 16 : (1 << (LOG2S % 4));   // first pass radix

    // S = 1024: the first pass (radix 32) writes at a stride of 32 values,
    // where the padding alone (one float2 per 16) still maps threads j and
    // j + 8 to the same banks.  Between the two passes logical element i is
    // therefore kept at pad16(i ^ ((i >> 8) & 1)): threads with bit 3 of j
    // set swap neighbouring values, which separates the two halves of a
    // half-warp; the second pass reads consecutive elements, which the swap
    // keeps within one 16-value line.
    static constexpr bool SWZ = S == 1024;
    static_assert(!SWZ || (T == 32 && R0 == 32 && NP == 2), "swizzled exchange layout");

    // PADDED_IN: the input sits at buf[pad16(i)] (else at buf[i]).
    // ZERO_HI: inputs S/2 .. S-1 are zero (a zero-padded transform): the
    // first pass neither reads them nor multiplies by them, so the caller
    // need not write them.  In the first pass thread j < S/R reads inputs
    // j + r S/R, which lie in the upper half exactly when r >= R/2.
    template <int SIGN, bool PADDED_IN, bool ZERO_HI = false>
    static __device__ __forceinline__ void run(float2* buf, float2* a, int t)
    {
        static_for<NP>([&](auto pp) {
            constexpr int p = decltype(pp)::value;
            constexpr int R = p == 0 ? R0 : V;
            constexpr int NS = p == 0 ? 1 : (V == 32 ? R0 : R0 * ipow16(p - 1));
            constexpr int C = V / R;
            constexpr bool LAST = p == NP - 1;
            static_for<C>([&](auto cc) {
                constexpr int c = decltype(cc)::value;
                const int j = t + c * T;
                const int pj = pad16(j);
                if constexpr (SWZ && p == 1) {
                    // element j + 32 r sits at pad16((j ^ ((r >> 3) & 1)) + 32 r)
                    const int pj1 = pad16(j ^ 1);
                    static_for<R>([&](auto rr) {
                        constexpr int r = decltype(rr)::value;
                        a[c * R + r] = buf[((r >> 3) & 1 ? pj1 : pj) + r * 34];
                    });
                } else {
                    static_for<R>([&](auto rr) {
                        constexpr int r = decltype(rr)::value;
                        if constexpr (ZERO_HI && p == 0 && r >= R / 2)
                            a[c * R + r] = make_float2(0.0f, 0.0f);
                        else
                            a[c * R + r] = buf[(p == 0 && !PADDED_IN) ? j + r * (S / R) : pad16_at<S / R>(j, pj, r)];
                    });
                }
            });
            __syncthreads();
            float dep = zero_after(a[0].x);
            static_for<C>([&](auto cc) {
                constexpr int c = decltype(cc)::value;
                const int j = t + c * T;
                const int jm = j % NS;
                float2* ar = a + c * R;
                if constexpr (p > 0)
                    apply_twiddle_powers<R>(ar, expi_pi<SIGN>(2.0f * (float)jm / (float)(NS * R) + dep));
                dft<R, SIGN>(ar);
                if constexpr (!LAST && SWZ) {
                    // element 32 j + r at pad16(32 j + (r ^ b)), b = bit 3 of j:
                    // 34 j + r + r / 16, plus b for even r and minus b for odd r
                    const int b = (j >> 3) & 1;
                    const int pe = 34 * j + b, po = 34 * j - b;
                    static_for<R>([&](auto rr) {
                        constexpr int r = decltype(rr)::value;
                        buf[(r & 1 ? po : pe) + r + (r >> 4)] = ar[r];
                    });
                } else if constexpr (!LAST) {
                    const int base = (j / NS) * NS * R + jm;
                    const int pb = pad16(base);
                    static_for<R>([&](auto rr) {
                        constexpr int r = decltype(rr)::value;
                        buf[pad16_at<NS>(base, pb, r)] = ar[r];
                    });
                }
                dep = zero_after(ar[R - 1].x);
            });
            if constexpr (!LAST) __syncthreads();
        });
    }
};

struct FourStepArgs {
    const void* v;                 // [B][D][L] io (first column kernel)
    const void* x[kMaxOrder];    // x_1..x_N, [B][D][L] io
    void* y;                       // [B][D][L] io
    const float2* H;               // [N][D][L] packed spectra (row kernel, conv mode)
    size_t H_bstride;              // slots between samples' spectra (0: shared by the batch)
    const float* bias;             // [N][D]
    float2* S;                     // scratch [wave][M1][M2] complex
    float2* Hout;                  // [rows][L] packed spectra (row kernel, spectrum mode)
    int B, D;
    int q0;                        // first sequence of the wave (channel-major index)
    int n;                         // order handled by this launch
    int n_last;                    // N - 1
};

template <int LOG2M1, int LOG2M2>
struct FourStep {
    static constexpr int M1 = 1 << LOG2M1, M2 = 1 << LOG2M2, M = M1 * M2;
    using F1 = SmemFft<LOG2M1>;
    using F2 = SmemFft<LOG2M2>;
    // row kernel: U units (row pairs) per CTA
    static constexpr int U = F2::T >= 128 ? 2 : 4;
    static constexpr int ROWS = 2 * U;
    static constexpr int ROW_THREADS = ROWS * F2::T;
    static constexpr int ROW_STRIDE = stride_mod16(M2, 2);
    static constexpr size_t ROW_SMEM = sizeof(float2) * ROWS * ROW_STRIDE;
    static constexpr int ROW_CTAS_PER_SEQ = (M1 / 2) / U;
    // column kernel: TC consecutive columns per CTA, column index fastest
    // across threads so every global access is a TC-element run (8 columns
    // at M1 = 1024, 64-byte runs, two CTAs per SM: 13 % slower on L = 2^20
    // than 16 columns with one CTA per SM)
    static constexpr int TC = (512 / F1::T) > 16 ? 16 : ((512 / F1::T) < 4 ? 4 : 512 / F1::T);
    static constexpr int COL_THREADS = TC * F1::T;
    static constexpr int COL_STRIDE = stride_mod16(M1, 16 / TC);
    static constexpr size_t COL_SMEM = sizeof(float2) * TC * COL_STRIDE;
    static constexpr int COL_CTAS_PER_SEQ = M2 / TC;
    static_assert(ROW_THREADS <= 1024 && COL_THREADS <= 1024, "block size");
    static_assert(ROW_SMEM <= 227 * 1024 && COL_SMEM <= 227 * 1024, "shared memory");
    static_assert(M2 % TC == 0 && (M1 / 2) % U == 0, "tiling");

    // Bin pairs (k, M - k) of the real split over the CTA's row pairs, in
    // shared memory after the forward row FFTs (row slot 2 up holds row u,
    // slot 2 up + 1 row M1 - u; unit 0: rows 0 and M1/2).  Thread tid takes
    // unit up = tid % U and k2 = tid / U + it KSTEP (it < ITER), so adjacent
    // threads touch adjacent spectrum slots (k1 consecutive), and the
    // split's twiddle exp(-i pi k / M) of iteration it is that of it = 0
    // times exp(-i pi it / ITER).  f(kind, p1, p2, k, w): kind 0 = bins k
    // (*p1) and M - k (*p2); 1 = bins 0 and M (slot 0, p1 == p2); 2 = bin
    // M/2 alone (p1 == p2).
    template <typename Fn>
    static __device__ __forceinline__ void for_each_pair(float2* smem, int ublk, int tid, Fn&& f)
    {
        constexpr int RS = ROW_STRIDE, KSTEP = ROW_THREADS / U, ITER = U * M2 / ROW_THREADS;
        constexpr int Q = 32 / ITER;          // exp(-i pi it / ITER) = W_64^(Q it)
        static_assert(ITER * KSTEP == M2 && 32 % ITER == 0, "pair iteration");
        const int up = tid % U, k20 = tid / U, u = ublk * U + up;
        float2* r0 = smem + (2 * up) * RS;
        float2* r1 = smem + (2 * up + 1) * RS;
        if (u != 0) {
            const int k0 = u + M1 * k20;                    // partner M - k: row M1 - u, slot M2 - 1 - k2
            const float2 w0 = expi_pi<-1>((float)k0 / (float)M);
            static_for<ITER>([&](auto ii) {
                constexpr int it = decltype(ii)::value;
                const int k2 = k20 + it * KSTEP;
                f(0, r0 + pad16(k2), r1 + pad16(M2 - 1 - k2), k0 + it * KSTEP * M1, mul_w64<Q * it, -1>(w0));
            });
        } else {
            // row M1/2 pairs with itself reversed; row 0 pairs k2 with M2 - k2
            const float2 wh0 = expi_pi<-1>((float)(M1 / 2 + M1 * k20) / (float)M);
            const float2 wz0 = expi_pi<-1>((float)(M1 * k20) / (float)M);
            static_for<ITER / 2>([&](auto ii) {
                constexpr int it = decltype(ii)::value;
                const int k2 = k20 + it * KSTEP;             // < M2 / 2
                f(0, r1 + pad16(k2), r1 + pad16(M2 - 1 - k2), M1 / 2 + M1 * k2, mul_w64<Q * it, -1>(wh0));
                if (k2 > 0) {
                    f(0, r0 + pad16(k2), r0 + pad16(M2 - k2), M1 * k2, mul_w64<Q * it, -1>(wz0));
                } else {
                    f(1, r0, r0, 0, make_float2(1.0f, 0.0f));
                    f(2, r0 + pad16(M2 / 2), r0 + pad16(M2 / 2), M / 2, make_float2(0.0f, -1.0f));
                }
            });
        }
    }

    // row of the CTA's row slot rr (units u: rows u and M1 - u; unit 0:
    // rows 0 and M1/2)
    static __device__ __forceinline__ int row_of(int ublk, int rr)
    {
        const int u = ublk * U + rr / 2;
        if (u == 0) return (rr & 1) ? M1 / 2 : 0;
        return (rr & 1) ? M1 - u : u;
    }
};

// The real split + bias-folded spectral multiply + inverse re-pack of one
// bin pair (k, Mtot - k), as in fused1d.cuh, in reduced form.  With
// z1 = Z[k], z2 = Z[Mtot - k] (the packed transform), w = exp(-i pi k /
// Mtot) = c + i s, the bias-folded filter bins G1 = (H[k] + b) / (2 Mtot),
// G2 = (H[Mtot - k] + b) / (2 Mtot), and P = G1 + conj(G2),
// Q = G1 - conj(G2) (the bias cancels in Q), the inverse transform's
// inputs are
//   Z'[k]        = (P + s Q) z1 + i c Q conj(z2),
//   Z'[Mtot - k] = conj(P - s Q) z2 + i c conj(Q) conj(z1):
// the split U[k] = ((z1 + conj z2) - i w (z1 - conj z2)) / 2 and its
// inverse re-pack composed, which leaves real coefficients 2 +- 2s and
// +-2ic on the products of (H + b) with z1 and conj(z2).
template <int MTOT>
__device__ __forceinline__ void spectral_pair(float2& z1, float2& z2, float2 h1, float2 h2,
                                              float2 w, float bias)
{
    constexpr float sc = 1.0f / (2.0f * (float)MTOT);
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

// The real split alone: packed spectrum bins k and Mtot - k from Z[k], Z[Mtot - k].
__device__ __forceinline__ void real_split(float2 z1, float2 z2, float2 w, float2& X1, float2& X2)
{
    const float2 bc = cconj(z2);
    const float2 S = cadd(z1, bc);
    const float2 Tw = cmul(w, csub(z1, bc));
    X1 = make_float2(0.5f * (S.x + Tw.y), 0.5f * (S.y - Tw.x));
    X2 = make_float2(0.5f * (S.x - Tw.y), -0.5f * (S.y + Tw.x));
}

// Row kernel.  SPECTRUM = false: one order of the forward (conv mode);
// SPECTRUM = true: forward row FFTs + real split written to Hout in the
// packed layout (filter spectra).
template <int LOG2M1, int LOG2M2, bool SPECTRUM>
__global__ void __launch_bounds__(FourStep<LOG2M1, LOG2M2>::ROW_THREADS)
fourstep_row_kernel(FourStepArgs a)
{
    grid_dependency_begin();
    using FS = FourStep<LOG2M1, LOG2M2>;
    constexpr int M1 = FS::M1, M2 = FS::M2, M = FS::M, U = FS::U, T2 = FS::F2::T, V2 = FS::F2::V;
    constexpr int RS = FS::ROW_STRIDE;
    extern __shared__ __align__(16) float2 smem_fs[];

    const int qi = blockIdx.x / FS::ROW_CTAS_PER_SEQ;        // sequence within the wave
    const int ublk = blockIdx.x % FS::ROW_CTAS_PER_SEQ;
    const int q = a.q0 + qi;                                 // channel-major index
    const int d = SPECTRUM ? 0 : q / a.B;
    float2* Sq = a.S + (size_t)qi * M;
    const int tid = threadIdx.x;

    // the wave scratch stays in L2 for the next launch; spectra and
    // activations stream through
    const uint64_t keep = l2_evict_last(), stream = l2_evict_first();
#pragma unroll 1
    for (int rr = 0; rr < FS::ROWS; ++rr)
        cp_async_row_hint(smem_fs + rr * RS, Sq + (size_t)FS::row_of(ublk, rr) * M2, M2 * 8, tid,
                          FS::ROW_THREADS, keep);
    cp_async_wait_all();
    __syncthreads();

    const int row = tid / T2, t = tid % T2;
    float2* rb = smem_fs + row * RS;
    float2 reg[V2];
    FS::F2::template run<-1, false>(rb, reg, t);
    const int pt = pad16(t);
    static_for<V2>([&](auto rr) {
        constexpr int r = decltype(rr)::value;
        rb[pad16_at<M2 / V2>(t, pt, r)] = reg[r];
    });
    __syncthreads();

    if constexpr (SPECTRUM) {
        float2* Ho = a.Hout + (size_t)q * M;
        FS::for_each_pair(smem_fs, ublk, tid, [&](int kind, float2* p1, float2* p2, int k, float2 w) {
            if (kind == 1) {                                    // bins 0 and M share slot 0
                const float2 z = *p1;
                st_hint(Ho, make_float2(z.x + z.y, z.x - z.y), stream);
            } else {
                float2 X1, X2;
                real_split(*p1, *p2, w, X1, X2);
                st_hint(Ho + k, X1, stream);
                if (kind == 0) st_hint(Ho + (M - k), X2, stream);
            }
        });
        return;
    } else {
        const float bias = __ldg(a.bias + a.n * a.D + d);
        const float2* Hr = a.H + (size_t)(q % a.B) * a.H_bstride + ((size_t)a.n * a.D + d) * M;
        FS::for_each_pair(smem_fs, ublk, tid, [&](int kind, float2* p1, float2* p2, int k, float2 w) {
            float2 z1 = *p1, z2 = *p2;
            if (kind == 1) {                                    // slot 0 holds (bin 0, bin M), both real
                const float2 h0 = ld_hint(Hr, stream);
                spectral_pair<M>(z1, z2, make_float2(h0.x, 0.0f), make_float2(h0.y, 0.0f), w, bias);
            } else {
                spectral_pair<M>(z1, z2, ld_hint(Hr + k, stream), ld_hint(Hr + (M - k), stream), w, bias);
            }
            *p1 = z1;
            if (kind == 0) *p2 = z2;
        });
        __syncthreads();

        FS::F2::template run<+1, true>(rb, reg, t);
        // B[k1][n2] *= exp(+2 pi i n2 k1 / M), n2 = t + r M2/V2
        const int k1 = FS::row_of(ublk, row);
        float2 w = expi_pi<+1>(2.0f * (float)((t * k1) % M) / (float)M);
        const float2 step = expi_pi<+1>(2.0f * (float)((k1 * (M2 / V2)) % M) / (float)M);
        static_for<V2>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            st_hint(Sq + (size_t)k1 * M2 + t + r * (M2 / V2), cmul(reg[r], w), keep);
            if constexpr (r < V2 - 1) w = cmul(w, step);
        });
    }
}

// Column kernel.  MODE 0: the first order's forward columns from v (or, for
// the spectrum, from h); MODE 1: inverse columns, gate, next order's forward
// columns; MODE 2: inverse columns, gate, store y.  PAD false: circular
// mode ("Handling Boundaries": periodic systems), the M-point transform of
// the unpadded sequence of 2M reals: every n1 is data and no output is
// cropped.
template <int LOG2M1, int LOG2M2, typename IO, int MODE, bool PAD = true>
__global__ void __launch_bounds__(FourStep<LOG2M1, LOG2M2>::COL_THREADS)
fourstep_col_kernel(FourStepArgs a)
{
    grid_dependency_begin();
    using FS = FourStep<LOG2M1, LOG2M2>;
    using IOP = IoPair<IO>;
    using PT = typename IOP::T;
    constexpr int M1 = FS::M1, M2 = FS::M2, M = FS::M, TC = FS::TC, V1 = FS::F1::V;
    constexpr int VL = PAD ? V1 / 2 : V1;                   // registers holding data (n1 < M1/2, or all)
    constexpr int SEQ = PAD ? M / 2 : M;                     // value pairs per sequence
    extern __shared__ __align__(16) float2 smem_fs[];

    const int qi = blockIdx.x / FS::COL_CTAS_PER_SEQ;
    const int c0 = (blockIdx.x % FS::COL_CTAS_PER_SEQ) * TC;
    const int q = a.q0 + qi;
    const int d = q / a.B, b = q % a.B;
    const size_t seq = (size_t)b * a.D + d;                  // (spectrum: a.B = 1, a.D = rows)
    float2* Sq = a.S + (size_t)qi * M;
    const int tid = threadIdx.x;
    const int c = tid % TC, t = tid / TC;
    const int n2 = c0 + c;
    float2* buf = smem_fs + c * FS::COL_STRIDE;
    float2 reg[V1];
    // the wave scratch stays in L2 for the next launch; activations stream
    const uint64_t keep = l2_evict_last(), stream = l2_evict_first();

    // float32 activations: the first order's columns of v straight into the
    // padded column buffers, two adjacent columns per 16-byte load
    constexpr bool VEC0 = MODE == 0 && std::is_same<IO, float>::value;
    if constexpr (VEC0) {
        constexpr int ROWS0 = PAD ? M1 / 2 : M1;                 // rows n1 holding data
        constexpr int RPP = FS::COL_THREADS / (TC / 2);
        static_assert(ROWS0 % RPP == 0, "column passes");
        const int cp = tid % (TC / 2), rr0 = tid / (TC / 2);
        float2* b0 = smem_fs + (2 * cp) * FS::COL_STRIDE;
        float2* b1 = b0 + FS::COL_STRIDE;
        const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float2*>(a.v) + seq * SEQ + c0 + 2 * cp);
        static_for<ROWS0 / RPP>([&](auto ii) {
            constexpr int i = decltype(ii)::value;
            const int n1 = rr0 + i * RPP;
            const float4 v = ld_hint4(src + (size_t)n1 * (M2 / 2), stream);
            b0[pad16(n1)] = make_float2(v.x, v.y);
            b1[pad16(n1)] = make_float2(v.z, v.w);
        });
    } else if constexpr (MODE == 0) {
        const PT* vp = reinterpret_cast<const PT*>(a.v) + seq * SEQ;
        static_for<VL>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            reg[r] = IOP::load_stream(vp + n2 + (size_t)M2 * (t + r * (M1 / V1)), stream);
        });
    } else {
        const void* xn = a.x[0];
#pragma unroll
        for (int i = 1; i < kMaxOrder; ++i)
            if (i == a.n) xn = a.x[i];
        const PT* xp = reinterpret_cast<const PT*>(xn) + seq * SEQ;
        // the CTA's TC columns of the scratch, two adjacent columns per
        // 16-byte load (a warp: 4 rows x 128 bytes), scattered into the
        // padded column buffers
        static_assert(TC % 2 == 0 && FS::COL_THREADS % (TC / 2) == 0, "column pairs");
        constexpr int RPP = FS::COL_THREADS / (TC / 2);           // rows per pass
        static_assert(M1 % RPP == 0, "column passes");
        {
            const int cp = tid % (TC / 2), rr0 = tid / (TC / 2);
            float2* b0 = smem_fs + (2 * cp) * FS::COL_STRIDE;
            float2* b1 = b0 + FS::COL_STRIDE;
            const float4* src = reinterpret_cast<const float4*>(Sq + c0 + 2 * cp);
            static_for<M1 / RPP>([&](auto ii) {
                constexpr int i = decltype(ii)::value;
                const int k1 = rr0 + i * RPP;
                const float4 v = ld_hint_rw4(src + (size_t)k1 * (M2 / 2), keep);
                b0[pad16(k1)] = make_float2(v.x, v.y);
                b1[pad16(k1)] = make_float2(v.z, v.w);
            });
        }
        __syncthreads();
        FS::F1::template run<+1, true>(buf, reg, t);
        // crop (n1 = t + r M1/V1 < M1/2 <=> r < V1/2; circular: none) and gate
        static_for<VL>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            const float2 xv = IOP::load_stream(xp + n2 + (size_t)M2 * (t + r * (M1 / V1)), stream);
            reg[r] = make_float2(reg[r].x * xv.x, reg[r].y * xv.y);
        });
        if constexpr (MODE == 2) {
            PT* yp = reinterpret_cast<PT*>(a.y) + seq * SEQ;
            static_for<VL>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                IOP::store_stream(yp + n2 + (size_t)M2 * (t + r * (M1 / V1)), reg[r], stream);
            });
            return;
        }
    }
    // forward column FFT of z (n1 < M1/2, zero-padded; circular: all n1),
    // then the four-step twiddle exp(-2 pi i n2 k1 / M)
    if constexpr (!VEC0) {
        const int pt = pad16(t);
        static_for<VL>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            buf[pad16_at<M1 / V1>(t, pt, r)] = reg[r];
        });
    }
    __syncthreads();
    FS::F1::template run<-1, true, PAD>(buf, reg, t);
    float2 w = expi_pi<-1>(2.0f * (float)((n2 * t) % M) / (float)M);
    const float2 step = expi_pi<-1>(2.0f * (float)((n2 * (M1 / V1)) % M) / (float)M);
    static_for<V1>([&](auto rr) {
        constexpr int r = decltype(rr)::value;
        st_hint(Sq + (size_t)(t + r * (M1 / V1)) * M2 + n2, cmul(reg[r], w), keep);
        if constexpr (r < V1 - 1) w = cmul(w, step);
    });
}

}  // namespace hyena
