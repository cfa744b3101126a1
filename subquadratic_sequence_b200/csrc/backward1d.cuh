// backward1d.cuh -- the backward pass of the single-CTA 1-D path (L <= 16384).
//
// The pages describe the forward only; its gradient follows from the chain
// rule.  With c_n = h_n (*) z_{n-1} + b_n z_{n-1} and z_n = x_n c_n, and
// g = dL/dz_n flowing back from g = dy at n = N:
//     dx_n        = g * c_n
//     e           = g * x_n                         (dL/dc_n)
//     dh_n[s]    += sum_t e[t] z_{n-1}[t - s]       (summed over the batch)
//     db_n       += sum_t e[t] z_{n-1}[t]  =  dh_n[0]
//     dz_{n-1}    = corr(h_n, e) + b_n e,   corr(h, e)[u] = sum_{t>=u} h[t-u] e[t]
// and dv = dz_0.  On the 2L-point grid (zero-padded, "Native
// Multi-Dimensional Subquadratic Operators via Input Dependent Long
// Convolutions", Handling Boundaries) both sums are correlations:
//     DFT(dz_{n-1}) = (conj(H_n) + b_n) DFT(e)          (first L outputs)
//     DFT(dh_n)     = sum_b DFT(e) conj(DFT(z_{n-1}))   (first L lags)
//
// One CTA group (T threads, the same FFT machinery and layouts as the fused
// forward) owns one unit (channel d, slice s of the batch) and walks the
// slice's sequences; the host picks the number of slices S so that the D S
// units fill the chip in the fewest rounds:
//   A. the forward again, saving Z_n = DFT(z_n) and c_{n+1} to the
//      workspace in register order (each thread reads back what it wrote);
//   B. for n = N..1: dx_n and e from g; E = DFT(e); accumulate E conj(Z)
//      into the unit's dh spectrum (only this group touches it, so a
//      plain read-modify-write; the slice's first sequence stores);
//      g = inverse of (conj(H_n) + b_n) E.
// Both phases run through one copy of the FFT code (a step loop), which
// halves the kernel's instruction footprint.  A second launch sums each
// channel's S slice spectra in slice order (deterministic), turns the sum
// into dh_n (inverse real FFT, first L lags) and db_n = dh_n[0].
//
// Per-sample filters (PS, input-dependent filters): sequence (b, d) reads
// sample b's spectra at H + b H_bstride, and its dh spectrum is its own
// (acc [B][N][D][L], no sum over the batch), so dh_n is per sample
// ([B][N][D][L]); the bias is shared, so db_n = sum_b dh_{b,n}[0].
//
// Circular mode (PAD = false, "Handling Boundaries": circular convolutions
// for periodic systems): the same steps on the L-point grid itself (L = 2M
// reals as M packed points, no padding, nothing cropped), so both sums are
// circular correlations and dh_n has all L lags.
#pragma once

#include "fused1d.cuh"

namespace hyena {

struct Backward1dArgs {
    const void* v;                 // [B][D][L] io
    const void* x[kMaxOrder];      // x_1..x_N, [B][D][L] io
    const void* dy;                // [B][D][L] io
    const float2* H;               // [N][D][L] packed filter spectra
    const float* bias;             // [N][D]
    void* dv;                      // [B][D][L] io
    void* dx[kMaxOrder];           // [B][D][L] io each
    float* dh;                     // [N][D][L]
    float* dbias;                  // [N][D]
    float2* acc;                   // workspace [S][N][D][L]: accumulated dh spectra (packed; [B][N][D][L] per sample)
    float2* wz;                    // workspace [S][D][N][L]: Z_n in register order
    float2* wc;                    // workspace [S][D][N][L/2]: c_{n+1} in register order
    int B, D, N;
    int S;                         // batch slices: unit u = s D + d takes samples [s B / S, (s + 1) B / S)
    size_t H_bstride;              // per-sample spectra: slots between samples' sets
};

template <int LOG2M, typename IO, bool PS = false, bool PAD = true>
__global__ void __launch_bounds__(Fft1d<LOG2M, PAD>::THREADS, Fft1d<LOG2M, PAD>::MIN_BLOCKS)
backward1d_kernel(Backward1dArgs args)
{
    grid_dependency_begin();
    using F = Fft1d<LOG2M, PAD>;
    using IOP = IoPair<IO>;
    using PT = typename IOP::T;
    constexpr int M = F::M, E = F::E, T = F::T, RF = F::P::RF;
    constexpr int SEQ = F::SEQ;                 // packed pairs per sequence: M/2 (padded), M (circular)
    constexpr int NIO = PAD ? E / 2 : E;        // io registers per thread
    // dh-spectrum update in three sweeps (loads batched ahead of stores)
    // except at M = 16384, where it would spill
    constexpr bool BATCH_ACC = LOG2M <= 13;
    extern __shared__ __align__(16) float2 smem_dyn[];

    const int g = threadIdx.x / T, t = threadIdx.x % T;
    const int D = args.D, N = args.N;
    const int units = D * args.S;
    const int u_raw = blockIdx.x * F::G + g;
    const bool active = u_raw < units;       // inactive groups compute but write nothing
    const int u = active ? u_raw : units - 1;
    const int sl = u / D, d = u - sl * D;    // slice, channel
    const int b0 = (int)((long)sl * args.B / args.S), b1 = (int)((long)(sl + 1) * args.B / args.S);
    float2* sm = smem_dyn + g * F::SMEM_SEQ;
    float2* stage = smem_dyn + F::G * F::SMEM_SEQ + g * F::STAGE_SEQ;
    float2* wz = args.wz + (size_t)u * N * M;
    float2* wc = args.wc + (size_t)u * N * SEQ;
    // index of io register i among the thread's NIO io registers
    auto io_slot = [](int i) { return PAD ? (i / RF) * (RF / 2) + i % RF : i; };
    auto pick = [](const void* const* arr, int n) {
        const void* p = arr[0];
#pragma unroll
        for (int i = 1; i < kMaxOrder; ++i)
            if (i == n) p = arr[i];
        return p;
    };

    float2 a[E];
    for (int b = b0; b < b1; ++b) {
        const size_t seq = (size_t)b * D + d;
        const float2* Hb = PS ? args.H + (size_t)b * args.H_bstride : args.H;
        {
            const PT* vp = reinterpret_cast<const PT*>(args.v) + seq * SEQ;
            F::for_each_io(t, [&](int i, int m) { a[i] = IOP::load(vp + m); });
        }
        // One step per order, forwards (A) and then backwards (B), through a
        // single FFT code path:
        //   A_n: a = z_n;  save Z_n = DFT(z_n);  c_{n+1} = inverse((H_n + b_n) Z_n),
        //        saved; a = x_{n+1} c_{n+1} (after the last order: a = dy)
        //   B_n: a = g;  dx_{n+1} = g c_{n+1};  a = e = g x_{n+1};  E = DFT(e);
        //        dh spectrum += E conj(Z_n);  a = g = inverse((conj H_n + b_n) E)
        for (int s = 0; s < 2 * N; ++s) {
            const bool back = s >= N;
            const int n = back ? 2 * N - 1 - s : s;
            const float bias = __ldg(args.bias + n * D + d);
            const PT* xp = reinterpret_cast<const PT*>(pick(args.x, n)) + seq * SEQ;
            float2* wcn = wc + (size_t)n * SEQ;
            if (back) {
                PT* dxp = reinterpret_cast<PT*>(const_cast<void*>(pick(reinterpret_cast<const void* const*>(args.dx), n)))
                          + seq * SEQ;
                // all loads first, then the stores: one latency, not one per value
                float2 c[NIO], xv[NIO];
                F::for_each_io(t, [&](int i, int m) {
                    c[io_slot(i)] = wcn[io_slot(i) * T + t];
                    xv[io_slot(i)] = IOP::load(xp + m);
                });
                F::for_each_io(t, [&](int i, int m) {
                    const int k = io_slot(i);
                    if (active) IOP::store(dxp + m, make_float2(a[i].x * c[k].x, a[i].y * c[k].y));
                    a[i] = make_float2(a[i].x * xv[k].x, a[i].y * xv[k].y);
                });
            }
            if constexpr (!F::H_IN_EXCHANGE)
                cp_async_row(stage, Hb + ((size_t)n * D + d) * M, M * 8, t, T);
            F::forward(a, sm, t);
            if (!back) {
                if (active)
                    static_for<E>([&](auto ii) {
                        constexpr int i = decltype(ii)::value;
                        wz[(size_t)n * M + i * T + t] = a[i];
                    });
            } else if (active) {
                // dh spectrum: acc[k] (+)= E[k] conj(Z_n[k]) over the 2L-point bins
                float2* acc = args.acc + (((size_t)(PS ? b : sl) * N + n) * D + d) * M;
                const float2* zr = wz + (size_t)n * M;
                const bool first = PS || b == b0;
                float2 z[E];
                static_for<E>([&](auto ii) {
                    constexpr int i = decltype(ii)::value;
                    z[i] = zr[i * T + t];
                });
                if constexpr (BATCH_ACC) {
                    // three sweeps so that the accumulator's loads are all issued
                    // before any of its stores (interleaved, each load would wait
                    // for the stores before it): the products, in place of z;
                    // the partial sums read back; the sums written
                    F::for_each_pair(t, [&](int i1, int i2, int k, int kind, float2 w) {
                        const float2 e1 = a[i1], e2 = a[i2];
                        if (kind == 1) {
                            // slot 0: bins 0 and M, both real
                            z[i1] = make_float2((e1.x + e1.y) * (z[i1].x + z[i1].y),
                                                (e1.x - e1.y) * (z[i1].x - z[i1].y));
                        } else {
                            float2 E1, E2, Z1, Z2;
                            split_pair(e1, e2, w, E1, E2);
                            split_pair(z[i1], z[i2], w, Z1, Z2);
                            z[i1] = cmulc(E1, Z1);
                            if (kind == 0) z[i2] = cmulc(E2, Z2);
                        }
                    });
                    if (!first)
                        F::for_each_pair(t, [&](int i1, int i2, int k, int kind, float2) {
                            z[i1] = cadd(z[i1], acc[k]);
                            if (kind == 0) z[i2] = cadd(z[i2], acc[M - k]);
                        });
                    F::for_each_pair(t, [&](int i1, int i2, int k, int kind, float2) {
                        acc[k] = z[i1];
                        if (kind == 0) acc[M - k] = z[i2];
                    });
                } else {
                    // one read-modify-write per pair (at L = 16384 the kernel
                    // runs at 128 registers and the sweeps above spill more
                    // than they save)
                    F::for_each_pair(t, [&](int i1, int i2, int k, int kind, float2 w) {
                        const float2 e1 = a[i1], e2 = a[i2];
                        if (kind == 1) {
                            const float2 p = make_float2((e1.x + e1.y) * (z[i1].x + z[i1].y),
                                                         (e1.x - e1.y) * (z[i1].x - z[i1].y));
                            acc[0] = first ? p : cadd(acc[0], p);
                        } else {
                            float2 E1, E2, Z1, Z2;
                            split_pair(e1, e2, w, E1, E2);
                            split_pair(z[i1], z[i2], w, Z1, Z2);
                            const float2 p1 = cmulc(E1, Z1);
                            acc[k] = first ? p1 : cadd(acc[k], p1);
                            if (kind == 0) {
                                const float2 p2 = cmulc(E2, Z2);
                                acc[M - k] = first ? p2 : cadd(acc[M - k], p2);
                            }
                        }
                    });
                }
            }
            const float2* Hs = stage;
            if constexpr (F::H_IN_EXCHANGE) {
                cp_async_row(sm, Hb + ((size_t)n * D + d) * M, M * 8, t, T);
                Hs = sm;
            }
            cp_async_wait_all();
            __syncthreads();                                  // H_n visible
            F::template spectral<false, true>(a, Hs, bias, t, back ? -1.0f : 1.0f);
            __syncthreads();                                  // H_n consumed
            F::inverse(a, sm, t);
            if (!back) {
                // a = c_{n+1}: save it, then z_{n+1} = x_{n+1} c_{n+1}, or g = dy
                const PT* gp = reinterpret_cast<const PT*>(args.dy) + seq * SEQ;
                F::for_each_io(t, [&](int i, int m) {
                    if (active) wcn[io_slot(i) * T + t] = a[i];
                    if (n + 1 < N) {
                        const float2 x = IOP::load(xp + m);
                        a[i] = make_float2(a[i].x * x.x, a[i].y * x.y);
                    } else {
                        a[i] = IOP::load(gp + m);
                    }
                });
            }
        }
        if (active) {
            PT* dvp = reinterpret_cast<PT*>(args.dv) + seq * SEQ;
            F::for_each_io(t, [&](int i, int m) { IOP::store(dvp + m, a[i]); });
        }
    }
}

// dh_n[d] and db_n[d] from the accumulated spectra: one group per row
// (n, d): the sum of the row's S slice spectra (in slice order), its
// inverse real FFT (scale 1/P), the first L lags, and db = dh[0].  PS: the
// group inverts the B per-sample spectra of its row in turn and db is the
// sum of their lag-0 values.
template <int LOG2M, bool PS = false, bool PAD = true>
__global__ void __launch_bounds__(Fft1d<LOG2M, PAD>::THREADS)
dh_finalize_kernel(Backward1dArgs args)
{
    grid_dependency_begin();
    using F = Fft1d<LOG2M, PAD>;
    constexpr int M = F::M, E = F::E, T = F::T;
    extern __shared__ __align__(16) float2 smem_dyn[];
    const int g = threadIdx.x / T, t = threadIdx.x % T;
    const int rows = args.N * args.D;
    const int row_raw = blockIdx.x * F::G + g;
    const bool active = row_raw < rows;
    const int row = active ? row_raw : rows - 1;
    float2* sm = smem_dyn + g * F::SMEM_SEQ;
    constexpr float s = 1.0f / (2.0f * (float)M);           // 1/P of the inverse DFT
    float db = 0.0f;
    for (int b = 0; b < (PS ? args.B : 1); ++b) {
    const size_t srow = (size_t)b * rows + row;              // [B][N][D] rows (b = 0 when shared)
    const float2* acc = args.acc + srow * M;
    const int nsl = PS ? 1 : args.S;                          // slice spectra [S][N][D] summed
    const size_t sstride = (size_t)rows * M;
    // the thread's bins (k in a[i1], M - k in a[i2]), summed over the slices
    // one slice at a time, so that each slice's loads go out together
    float2 a[E];
    F::for_each_pair(t, [&](int i1, int i2, int k, int kind, float2) {
        a[i1] = acc[k];
        if (kind == 0) a[i2] = acc[M - k];
    });
    for (int q = 1; q < nsl; ++q) {
        const float2* aq = acc + q * sstride;
        F::for_each_pair(t, [&](int i1, int i2, int k, int kind, float2) {
            a[i1] = cadd(a[i1], aq[k]);
            if (kind == 0) a[i2] = cadd(a[i2], aq[M - k]);
        });
    }
    F::for_each_pair(t, [&](int i1, int i2, int k, int kind, float2 w) {
        float2 z1, z2;
        if (kind == 1) {
            const float2 p = a[i1];                           // slot 0: bins 0 and M
            unsplit_pair(make_float2(p.x, 0.0f), make_float2(p.y, 0.0f), w, s, z1, z2);
            a[i1] = z1;
        } else if (kind == 2) {
            const float2 y = a[i1];
            unsplit_pair(y, y, w, s, z1, z2);
            a[i1] = z1;
        } else {
            unsplit_pair(a[i1], a[i2], w, s, z1, z2);
            a[i1] = z1;
            a[i2] = z2;
        }
    });
    F::inverse(a, sm, t);
    if (active) {
        float2* dhp = reinterpret_cast<float2*>(args.dh) + srow * F::SEQ;   // L = 2 SEQ lags a row
        F::for_each_io(t, [&](int i, int m) {
            dhp[m] = a[i];
            if (m == 0) db += a[i].x;                         // db_n = sum of dh_n[0]
        });
    }
    __syncthreads();                                          // sm is reused by the next sample
    }
    if (active)
        F::for_each_io(t, [&](int i, int m) {
            if (m == 0) args.dbias[row] = db;
        });
}

}  // namespace hyena
