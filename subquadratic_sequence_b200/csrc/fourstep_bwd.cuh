// fourstep_bwd.cuh -- the backward pass of the four-step (long L) path.
//
// The chain rule of the recurrence, as for the single-CTA backward (the
// pages give the forward only): with c_n = h_n (*) z_n + b_n z_n,
// z_{n+1} = x_n c_n and g = dL/dz_{n+1} (dy for the last order),
//     dx_n = g c_n,   e = g x_n,
//     DFT(dh_n) += E conj(Z_n)           (summed over the batch; lags < L)
//     db_n = dh_n[0]
//     DFT(g)     = (conj(H_n) + b_n) E   (outputs < L)
// on the 2L-point grid ("Native Multi-Dimensional Subquadratic Operators
// via Input Dependent Long Convolutions", Handling Boundaries).  The
// M = L-point complex transform of the packed sequence runs as the forward
// does: M1-point columns (twiddled) and M2-point rows, the real split over
// bin pairs (k, M - k) in the row step.
//
// Per wave of sequences:
//   A. the forward again: columns of v; per order the row step saving the
//      row-transformed spectrum Zc of z_n (before the split), and the
//      column step saving c_n and (but for the last order) gating and
//      transforming z_{n+1};
//   B. per order n = N-1 .. 0: columns: g (dy, or the inverse columns of
//      the scratch), dx_n, e = g x_n, forward columns of e; rows, one CTA
//      per (channel, row pair block) over the channel's sequences in the
//      wave: forward rows of e, the saved Zc rows beside them, per bin
//      pair the split of both, dh spectrum += E conj(Z) (only this CTA
//      touches those bins), the multiply by conj(H_n) + b_n and the
//      re-pack, inverse rows;
//   then the inverse columns of the scratch give dv.
// After the last wave each accumulated spectrum (packed like the filter
// spectra) is re-packed, inverse-transformed by rows and columns, and
// cropped: dh_n, and db_n = dh_n[0].
//
// Per-sample spectra (f.H_bstride != 0, input-dependent filters): sequence
// (b, d) reads sample b's H and owns its own dh spectrum (acc [B][N][D][M]),
// so dh is [B][N][D][L]; the shared bias's db_n = sum_b dh_{b,n}[0] is
// summed by a last small launch.
#pragma once

#include "fourstep.cuh"

namespace hyena {

struct FourStepBwdArgs {
    FourStepArgs f;                // v, x, H, bias, S (scratch), B, D, q0, n
    const void* dy;                // [B][D][L] io
    void* dv;                      // [B][D][L] io
    void* dx[kMaxOrder];           // [B][D][L] io each
    float2* zsave;                 // [N][wcap][M1][RS] row-transformed spectra of z_n, rows in the
                                   // padded shared-memory layout (RS = the row kernel's row stride)
    float2* csave;                 // [N][wcap][M/2] c_n (value pairs)
    float2* acc;                   // [N][D][M] accumulated dh spectra (packed like H); [B][N][D][M]
                                   // with per-sample spectra
    float* dh;                     // [N][D][L] ([B][N][D][L] with per-sample spectra)
    float* dbias;                  // [N][D]
    int wcap;                      // sequences a wave holds
    int nq;                        // sequences (or filter rows) in this wave
    int first;                     // columns MODE 1: g = dy
    int last;                      // columns MODE 0: the last order (save c_n only)
};

// The re-pack of a bin pair's spectrum values Y1 = Y[k], Y2 = Y[M - k]
// (already scaled by 1/2M) into the complex transform's bins k and M - k.
__device__ __forceinline__ void repack_pair(float2 Y1, float2 Y2, float2 w, float2& z1, float2& z2)
{
    const float2 U = make_float2(Y1.x + Y2.x, Y1.y - Y2.y);
    const float2 V = cmulc(make_float2(Y1.x - Y2.x, Y1.y + Y2.y), w);
    z1 = make_float2(U.x - V.y, U.y + V.x);
    z2 = make_float2(U.x + V.y, V.x - U.y);
}

template <typename T>
__device__ __forceinline__ T pick_fs(T const* arr, int n)
{
    T p = arr[0];
#pragma unroll
    for (int i = 1; i < kMaxOrder; ++i)
        if (i == n) p = arr[i];
    return p;
}

template <int LOG2M1, int LOG2M2>
struct FourStepBwd {
    using FS = FourStep<LOG2M1, LOG2M2>;
    // rows of e, then (MODE 1) the saved rows of Zc at a fixed offset
    static constexpr int ZOFF = FS::ROWS * FS::ROW_STRIDE;
    static constexpr size_t ROW_SMEM_B = 2 * FS::ROW_SMEM;
};

// Row kernel of the backward.  MODE 0 (A): the forward row step of order
// n, with the row-transformed rows saved to zsave[n].  MODE 1 (B): per
// (channel, row-pair block) over the channel's sequences in the wave (see
// above).  MODE 2: per filter row q of the accumulated spectra: re-pack,
// inverse rows, inverse twiddle into the scratch.
template <int LOG2M1, int LOG2M2, int MODE>
__global__ void __launch_bounds__(FourStep<LOG2M1, LOG2M2>::ROW_THREADS)
fourstep_bwd_row_kernel(FourStepBwdArgs ba)
{
    grid_dependency_begin();
    const FourStepArgs& a = ba.f;
    using FS = FourStep<LOG2M1, LOG2M2>;
    using FB = FourStepBwd<LOG2M1, LOG2M2>;
    constexpr int M1 = FS::M1, M2 = FS::M2, M = FS::M, T2 = FS::F2::T, V2 = FS::F2::V;
    constexpr int RS = FS::ROW_STRIDE;
    extern __shared__ __align__(16) float2 smem_fb[];
    const int ublk = blockIdx.x % FS::ROW_CTAS_PER_SEQ;
    const int unit = blockIdx.x / FS::ROW_CTAS_PER_SEQ;       // sequence (A), channel (B), filter row (2)
    const int tid = threadIdx.x;
    const int row = tid / T2, t = tid % T2;
    float2* rb = smem_fb + row * RS;
    const int k1 = FS::row_of(ublk, row);
    float2 reg[V2];
    const int pt = pad16(t);

    // inverse row transform of the CTA's rows, inverse twiddle
    // exp(+2 pi i n2 k1 / M), store into rows k1 of Sq
    auto inverse_rows = [&](float2* Sq) {
        FS::F2::template run<+1, true>(rb, reg, t);
        float2 w = expi_pi<+1>(2.0f * (float)((t * k1) % M) / (float)M);
        const float2 step = expi_pi<+1>(2.0f * (float)((k1 * (M2 / V2)) % M) / (float)M);
        static_for<V2>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            Sq[(size_t)k1 * M2 + t + r * (M2 / V2)] = cmul(reg[r], w);
            if constexpr (r < V2 - 1) w = cmul(w, step);
        });
    };
    // the CTA's rows of a sequence's scratch (row length M2, at 0) or of its
    // saved spectrum (padded rows of RS, at ZOFF) into shared memory
    auto stage_rows = [&](const float2* src, int off, int len) {
#pragma unroll 1
        for (int rr = 0; rr < FS::ROWS; ++rr)
            cp_async_row(smem_fb + off + rr * RS, src + (size_t)FS::row_of(ublk, rr) * len, len * 8, tid,
                         FS::ROW_THREADS);
    };
    // forward row transform of the CTA's rows, in natural order back to
    // shared memory (padded) and, if given, to zs in the same layout
    auto forward_rows = [&](float2* zs) {
        FS::F2::template run<-1, false>(rb, reg, t);
        static_for<V2>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            const int pk = pad16_at<M2 / V2>(t, pt, r);
            rb[pk] = reg[r];
            if (zs) zs[(size_t)k1 * RS + pk] = reg[r];
        });
        __syncthreads();
    };

    if constexpr (MODE == 2) {
        const int q = a.q0 + unit;                                // filter row n*D + d
        const float2* Ar = ba.acc + (size_t)q * M;
        float2* Sq = a.S + (size_t)unit * M;
        constexpr float s = 1.0f / (2.0f * (float)M);            // 1/P of the inverse
        FS::for_each_pair(smem_fb, ublk, tid, [&](int kind, float2* p1, float2* p2, int k, float2 w) {
            float2 z1, z2;
            if (kind == 1) {                                      // slot 0: bins 0 and M, both real
                const float2 a0 = Ar[0];
                repack_pair(make_float2(a0.x * s, 0.0f), make_float2(a0.y * s, 0.0f), w, z1, z2);
            } else {
                const float2 y1 = Ar[k], y2 = Ar[M - k];
                repack_pair(make_float2(y1.x * s, y1.y * s), make_float2(y2.x * s, y2.y * s), w, z1, z2);
            }
            *p1 = z1;
            if (kind == 0) *p2 = z2;
        });
        __syncthreads();
        inverse_rows(Sq);
        return;
    } else if constexpr (MODE == 0) {
        const int qi = unit, q = a.q0 + qi;
        const int d = q / a.B;
        float2* Sq = a.S + (size_t)qi * M;
        stage_rows(Sq, 0, M2);
        cp_async_wait_all();
        __syncthreads();
        forward_rows(ba.zsave + ((size_t)a.n * ba.wcap + qi) * M1 * RS);
        const float bias = __ldg(a.bias + a.n * a.D + d);
        const float2* Hr = a.H + (size_t)(q % a.B) * a.H_bstride + ((size_t)a.n * a.D + d) * M;
        FS::for_each_pair(smem_fb, ublk, tid, [&](int kind, float2* p1, float2* p2, int k, float2 w) {
            float2 z1 = *p1, z2 = *p2;
            if (kind == 1) {
                const float2 h0 = __ldg(Hr);
                spectral_pair<M>(z1, z2, make_float2(h0.x, 0.0f), make_float2(h0.y, 0.0f), w, bias);
            } else {
                spectral_pair<M>(z1, z2, __ldg(Hr + k), __ldg(Hr + (M - k)), w, bias);
            }
            *p1 = z1;
            if (kind == 0) *p2 = z2;
        });
        __syncthreads();
        inverse_rows(Sq);
    } else {
        const int d = a.q0 / a.B + unit;
        const int qa = max(a.q0, d * a.B), qb = min(a.q0 + ba.nq, (d + 1) * a.B);
        const float bias = __ldg(a.bias + a.n * a.D + d);
        const bool ps = a.H_bstride != 0;
        for (int q = qa; q < qb; ++q) {
            const int qi = q - a.q0;
            // per-sample spectra: sample b's H and its own dh spectrum
            const size_t sb = ps ? (size_t)(q % a.B) : 0;
            const float2* Hr = a.H + sb * a.H_bstride + ((size_t)a.n * a.D + d) * M;
            float2* Ar = ba.acc + ((sb * (a.n_last + 1) + a.n) * a.D + d) * M;
            float2* Sq = a.S + (size_t)qi * M;
            stage_rows(Sq, 0, M2);
            stage_rows(ba.zsave + ((size_t)a.n * ba.wcap + qi) * M1 * RS, FB::ZOFF, RS);
            cp_async_wait_all();
            __syncthreads();
            forward_rows(nullptr);                                // E (rows of e)
            // the products E conj(Z) replace the staged Z rows, then the
            // accumulator is read in one sweep and written in another, so
            // its loads are not each held behind the previous store (every
            // thread touches only its own pairs: no barrier in between)
            FS::for_each_pair(smem_fb, ublk, tid, [&](int kind, float2* p1, float2* p2, int k, float2 w) {
                const float2 e1 = *p1, e2 = *p2, y1 = p1[FB::ZOFF], y2 = p2[FB::ZOFF];
                float2 z1 = e1, z2 = e2;
                if (kind == 1) {
                    // slot 0: bins 0 and M, both real
                    p1[FB::ZOFF] = make_float2((e1.x + e1.y) * (y1.x + y1.y), (e1.x - e1.y) * (y1.x - y1.y));
                    const float2 h0 = __ldg(Hr);
                    spectral_pair<M>(z1, z2, make_float2(h0.x, 0.0f), make_float2(h0.y, 0.0f), w, bias);
                } else {
                    float2 E1, E2, Z1, Z2;
                    real_split(e1, e2, w, E1, E2);
                    real_split(y1, y2, w, Z1, Z2);
                    p1[FB::ZOFF] = cmulc(E1, Z1);
                    if (kind == 0) p2[FB::ZOFF] = cmulc(E2, Z2);
                    spectral_pair<M>(z1, z2, cconj(__ldg(Hr + k)), cconj(__ldg(Hr + (M - k))), w, bias);
                }
                *p1 = z1;
                if (kind == 0) *p2 = z2;
            });
            FS::for_each_pair(smem_fb, ublk, tid, [&](int kind, float2* p1, float2* p2, int k, float2) {
                p1[FB::ZOFF] = cadd(p1[FB::ZOFF], Ar[k]);
                if (kind == 0) p2[FB::ZOFF] = cadd(p2[FB::ZOFF], Ar[M - k]);
            });
            FS::for_each_pair(smem_fb, ublk, tid, [&](int kind, float2* p1, float2* p2, int k, float2) {
                Ar[k] = p1[FB::ZOFF];
                if (kind == 0) Ar[M - k] = p2[FB::ZOFF];
            });
            __syncthreads();
            inverse_rows(Sq);
        }
    }
}

// Column kernel of the backward (PAD false: circular mode, every n1 is data
// and nothing is cropped).  Each CTA: TC columns n2 of one sequence
// (one filter row in MODE 3).  MODE 0 (A): inverse columns, crop: c_n,
// saved; unless last, gate with x_n and forward columns + twiddle.  MODE 1
// (B): g = dy (first) or the inverse columns of the scratch; dx_n = g c_n;
// e = g x_n; forward columns + twiddle.  MODE 2: dv = the inverse columns.
// MODE 3: dh = the inverse columns of the finalize scratch, db = dh[0].
template <int LOG2M1, int LOG2M2, typename IO, int MODE, bool PAD = true>
__global__ void __launch_bounds__(FourStep<LOG2M1, LOG2M2>::COL_THREADS)
fourstep_bwd_col_kernel(FourStepBwdArgs ba)
{
    grid_dependency_begin();
    const FourStepArgs& a = ba.f;
    using FS = FourStep<LOG2M1, LOG2M2>;
    using IOP = IoPair<IO>;
    using PT = typename IOP::T;
    constexpr int M1 = FS::M1, M2 = FS::M2, M = FS::M, TC = FS::TC, V1 = FS::F1::V;
    constexpr int VL = PAD ? V1 / 2 : V1;                   // registers holding data (circular: all n1)
    constexpr int SEQ = PAD ? M / 2 : M;                     // value pairs per sequence
    extern __shared__ __align__(16) float2 smem_fc[];

    const int qi = blockIdx.x / FS::COL_CTAS_PER_SEQ;
    const int c0 = (blockIdx.x % FS::COL_CTAS_PER_SEQ) * TC;
    const int q = a.q0 + qi;
    const int d = q / a.B, b = q % a.B;
    const size_t seq = (size_t)b * a.D + d;
    float2* Sq = a.S + (size_t)qi * M;
    const int tid = threadIdx.x;
    const int c = tid % TC, t = tid / TC;
    const int n2 = c0 + c;
    float2* buf = smem_fc + c * FS::COL_STRIDE;
    const int pt = pad16(t);
    float2 reg[V1];
    // element n1 = t + r M1/V1 (r < V1/2) of column n2 is value pair m = n1 M2 + n2
    auto at = [&](int r) { return (size_t)M2 * (t + r * (M1 / V1)) + n2; };

    // inverse columns of the scratch, cropped to n1 < M1/2 (in reg[r], r <
    // V1/2); the transform's last pass reads buf before a barrier, so buf
    // may be written again as soon as it returns
    auto inverse_cols = [&]() {
        static_for<V1>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            buf[pad16_at<M1 / V1>(t, pt, r)] = Sq[(size_t)(t + r * (M1 / V1)) * M2 + n2];
        });
        __syncthreads();
        FS::F1::template run<+1, true>(buf, reg, t);
    };

    if constexpr (MODE == 3) {
        // q: filter row n*D + d; dh row of L floats = M/2 value pairs
        inverse_cols();
        float2* dhp = reinterpret_cast<float2*>(ba.dh) + (size_t)q * SEQ;
        static_for<VL>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            dhp[at(r)] = reg[r];
        });
        if (n2 == 0 && t == 0 && a.H_bstride == 0) ba.dbias[q] = reg[0].x;   // db_n = dh_n[0]
        return;
    } else {
        const size_t cso = ((size_t)a.n * ba.wcap + qi) * SEQ;
        float2* cs = ba.csave + cso;
        const PT* xp = reinterpret_cast<const PT*>(pick_fs(a.x, a.n)) + seq * SEQ;
        if constexpr (MODE == 0) {
            inverse_cols();                                     // c_n
            static_for<VL>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                cs[at(r)] = reg[r];
            });
            if (ba.last) return;
            static_for<VL>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                const float2 xv = IOP::load(xp + at(r));
                reg[r] = make_float2(reg[r].x * xv.x, reg[r].y * xv.y);
            });
        } else if constexpr (MODE == 1) {
            if (ba.first) {
                const PT* gp = reinterpret_cast<const PT*>(ba.dy) + seq * SEQ;
                static_for<VL>([&](auto rr) {
                    constexpr int r = decltype(rr)::value;
                    reg[r] = IOP::load(gp + at(r));
                });
            } else {
                inverse_cols();                                 // g = dL/dz_{n+1}
            }
            PT* dxp = reinterpret_cast<PT*>(pick_fs(ba.dx, a.n)) + seq * SEQ;
            float2 cv[VL], xv[VL];
            static_for<VL>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                cv[r] = cs[at(r)];
                xv[r] = IOP::load(xp + at(r));
            });
            static_for<VL>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                IOP::store(dxp + at(r), make_float2(reg[r].x * cv[r].x, reg[r].y * cv[r].y));
                reg[r] = make_float2(reg[r].x * xv[r].x, reg[r].y * xv[r].y);     // e
            });
        } else {
            inverse_cols();                                     // dv = dL/dz_0
            PT* dvp = reinterpret_cast<PT*>(ba.dv) + seq * SEQ;
            static_for<VL>([&](auto rr) {
                constexpr int r = decltype(rr)::value;
                IOP::store(dvp + at(r), reg[r]);
            });
            return;
        }
        // forward columns (n1 < M1/2, zero-padded; circular: all n1) + twiddle exp(-2 pi i n2 k1 / M)
        static_for<VL>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            buf[pad16_at<M1 / V1>(t, pt, r)] = reg[r];
        });
        __syncthreads();
        FS::F1::template run<-1, true, PAD>(buf, reg, t);
        float2 w = expi_pi<-1>(2.0f * (float)((n2 * t) % M) / (float)M);
        const float2 step = expi_pi<-1>(2.0f * (float)((n2 * (M1 / V1)) % M) / (float)M);
        static_for<V1>([&](auto rr) {
            constexpr int r = decltype(rr)::value;
            Sq[(size_t)(t + r * (M1 / V1)) * M2 + n2] = cmul(reg[r], w);
            if constexpr (r < V1 - 1) w = cmul(w, step);
        });
    }
}

// Per-sample spectra: db_n[d] = sum_b dh_{b,n}[d][0] over dh rows of L
// floats, one thread per (n, d), the samples in order (deterministic).
template <int L>
__global__ void __launch_bounds__(256) dbias_sum_kernel(FourStepBwdArgs ba)
{
    grid_dependency_begin();
    const int rows = (ba.f.n_last + 1) * ba.f.D;
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    float s = 0.0f;
    for (int b = 0; b < ba.f.B; ++b) s += ba.dh[((size_t)b * rows + r) * L];
    ba.dbias[r] = s;
}

}  // namespace hyena
