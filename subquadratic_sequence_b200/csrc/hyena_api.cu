// hyena_api.cu -- the extern "C" entry points declared in include/hyena.h:
// argument validation on the host, then the dispatchers of launch.cuh.
#include <stdint.h>

#include "k_circular.cuh"
#include "k_fft2d.cuh"
#include "k_fft2d_bwd.cuh"
#include "k_fourstep.cuh"
#include "k_fourstep_bwd.cuh"
#include "k_fft3d.cuh"
#include "k_fft3d_bwd.cuh"
#include "launch.cuh"

using namespace hyena;

namespace {

thread_local int g_last_cuda_error = 0;

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// [a, a + na) and [b, b + nb) share a byte
bool overlap(const void* a, size_t na, const void* b, size_t nb)
{
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + nb && b0 < a0 + na;
}

int exact_log2(long n)
{
    if (n <= 0 || (n & (n - 1)) != 0) return -1;
    int k = 0;
    while ((1L << k) < n) ++k;
    return k;
}

size_t io_bytes(hyena_dtype_t io) { return io == HYENA_BF16 ? 2 : 4; }

size_t scratch_bytes(long nseq, long L) { return sizeof(float2) * (size_t)wave_seqs(nseq, L) * L; }

// spectra of rows filters: single-CTA kernel or four-step (scratch needed)
hyena_status_t spectra(int log2m, const float* h, int rows, float2* H, float2* scratch,
                       cudaStream_t st)
{
    if (log2m <= kMaxLog2Fused) {
        Rfft1dArgs ra;
        ra.h = h;
        ra.H = H;
        ra.rows = rows;
        return dispatch_rfft(log2m, ra, st);
    }
    return dispatch_fourstep_rfft(log2m, h, rows, H, scratch, st);
}

// Validates a 1-D length: INVALID_ARG for L < 1, UNSUPPORTED outside the
// implemented set (powers of two in [16, 2^max_log2]).
hyena_status_t check_len(long L, int max_log2, int* log2m)
{
    if (L < 1) return HYENA_ERR_INVALID_ARG;
    const int k = exact_log2(L);
    if (k < kMinLog2 || k > max_log2) return HYENA_ERR_UNSUPPORTED;
    *log2m = k;
    return HYENA_OK;
}

hyena_status_t check_ffn(const hyena_ffn_t* f)
{
    if (!f || !f->W1 || !f->W2 || !f->W3 || !f->Wout || !f->alpha) return HYENA_ERR_INVALID_ARG;
    if (f->width < 1 || f->n_bands < 0 || !(f->decay_div > 0.0f)) return HYENA_ERR_INVALID_ARG;
    if (f->width > kFfnWidth || f->n_bands > 16) return HYENA_ERR_UNSUPPORTED;
    const void* w[5] = {f->W1, f->W2, f->W3, f->Wout, f->alpha};
    for (const void* p : w)
        if (!aligned(p, 4)) return HYENA_ERR_INVALID_ARG;
    return HYENA_OK;
}

hyena_status_t filter_gen(const hyena_ffn_t* f, int rows, int D, long npos, int L, int Hh,
                          int Ww, bool two_d, float* h, cudaStream_t st,
                          const hyena_film_t* film = nullptr, int B = 1, int Zz = 0)
{
    FilterGenArgs a = {};
    a.W1 = f->W1; a.W2 = f->W2; a.W3 = f->W3; a.Wout = f->Wout; a.alpha = f->alpha;
    a.n_in = !two_d ? 1 + 2 * f->n_bands : (Zz ? 3 + 6 * f->n_bands : 2 + 4 * f->n_bands);
    a.Zz = Zz;
    a.inv_Z = Zz > 0 ? 1.0f / (float)Zz : 0.0f;
    a.width = f->width;
    a.rows = rows;
    a.D = D;
    a.L = L; a.Hh = Hh; a.Ww = Ww;
    a.n_bands = f->n_bands;
    a.inv_div = 1.0f / f->decay_div;
    a.h = h;
    a.vec = (npos % 4 == 0 && aligned(h, 16)) ? 1 : 0;
    a.sample_stride = (long)rows * npos;
    a.inv_L = L > 0 ? 1.0f / (float)L : 0.0f;
    a.inv_H = Hh > 0 ? 1.0f / (float)Hh : 0.0f;
    a.inv_W = Ww > 0 ? 1.0f / (float)Ww : 0.0f;
    if (film) {
        a.omega = film->omega;
        a.gamma = film->gamma;
        a.beta = film->beta;
        a.film = (film->omega || film->gamma || film->beta) ? 1 : 0;
        if (film->sigma) {
            a.gaussian = 1;
            a.alpha = film->sigma;                 // the per-channel window parameter
        }
    }
    return launch_filter_gen(a, two_d, npos, B, st);
}

// packed spectrum: L complex slots per filter (bins 0 and L share slot 0)
size_t spectrum_bytes(long N, long D, long L) { return sizeof(float2) * N * D * L; }

size_t round_up(size_t n, size_t a) { return (n + a - 1) / a * a; }

// Workspace of the single-CTA backward (L <= 16384): per batch slice (at
// most min(B, 8) of them) a dh spectrum set acc [S][N][D][M] (per sample:
// [B][N][D][M]) and the saved Z_n (wz) and c_n (wc) of each unit.  M = L
// packed slots (L/2 circular); c_n takes half of that (all of it circular).
struct Bwd1dLayout {
    size_t acc, wz, wc, total;
    int slices;
};

Bwd1dLayout bwd1d_layout(int B, int D, int L, int N, bool per_sample, bool circular)
{
    constexpr int kMaxBwdSlices = 8;
    Bwd1dLayout l;
    l.slices = B < kMaxBwdSlices ? B : kMaxBwdSlices;
    const size_t spec = sizeof(float2) * (size_t)N * D * (circular ? L / 2 : L);   // one spectrum set
    const size_t cset = circular ? spec : spec / 2;
    l.acc = 0;
    l.wz = round_up(spec * (per_sample ? (size_t)B : (size_t)l.slices), 256);
    l.wc = l.wz + round_up(spec * l.slices, 256);
    l.total = l.wc + round_up(cset * l.slices, 256);
    return l;
}

hyena_status_t forward_impl(const void* v, const void* const* x, const float* h, const float* H,
                            bool per_sample, const float* bias, int B, int D, int L, int N,
                            hyena_dtype_t io, void* y, void* workspace, size_t ws_bytes, void* stream);
hyena_status_t forward2d_impl(const void* v, const void* const* x, const float* h, const float* Hs,
                              bool per_sample, const float* bias, int B, int C, int H, int W, int N,
                              hyena_dtype_t io, void* y, void* workspace, size_t ws_bytes, void* stream);
hyena_status_t backward_impl(const void* v, const void* const* x, const float* H, bool per_sample,
                             bool circular, const float* bias, const void* dy, int B, int D, int L, int N,
                             hyena_dtype_t io, void* dv, void* const* dx, float* dh, float* dbias,
                             void* workspace, size_t ws_bytes, void* stream);
hyena_status_t backward2d_impl(const void* v, const void* const* x, const float* Hs, bool per_sample,
                               bool circular, const float* bias, const void* dy, int B, int C, int H, int W,
                               int N, hyena_dtype_t io, void* dv, void* const* dx, float* dh, float* dbias,
                               void* workspace, size_t ws_bytes, void* stream);
bool dims2d_circ_ok(int H, int W, int& lh, int& lm);
hyena_status_t forward3d_impl(const void* v, const void* const* x, const float* h, const float* Hs,
                              bool per_sample, const float* bias, int B, int C, int Z, int H, int W,
                              int N, hyena_dtype_t io, void* y, void* workspace, size_t ws_bytes,
                              void* stream);

}  // namespace

namespace hyena {
hyena_status_t from_cuda(cudaError_t e)
{
    if (e == cudaSuccess) return HYENA_OK;
    g_last_cuda_error = (int)e;
    return HYENA_ERR_CUDA;
}
}  // namespace hyena

extern "C" {

const char* hyena_status_string(hyena_status_t s)
{
    switch (s) {
    case HYENA_OK: return "HYENA_OK";
    case HYENA_ERR_INVALID_ARG: return "HYENA_ERR_INVALID_ARG: invalid argument";
    case HYENA_ERR_UNSUPPORTED: return "HYENA_ERR_UNSUPPORTED: shape or option not implemented";
    case HYENA_ERR_WORKSPACE: return "HYENA_ERR_WORKSPACE: workspace missing or too small";
    case HYENA_ERR_CUDA: return "HYENA_ERR_CUDA: a CUDA call failed";
    }
    return "unknown hyena_status_t";
}

int hyena_last_cuda_error(void) { return g_last_cuda_error; }

hyena_status_t hyena_filter_gen(const hyena_ffn_t* ffn, int N, int D, int L, float* h, void* stream)
{
    hyena_status_t s = check_ffn(ffn);
    if (s != HYENA_OK) return s;
    if (!h || N < 1 || D < 1 || L < 1 || !aligned(h, 4)) return HYENA_ERR_INVALID_ARG;
    if ((long)N * D > 65535L * kFgRowTile || (long)N * D * (long)L > (1L << 40))
        return HYENA_ERR_UNSUPPORTED;
    return filter_gen(ffn, N * D, D, L, L, 0, 0, false, h, (cudaStream_t)stream);
}

hyena_status_t hyena_filter_gen_film(const hyena_ffn_t* ffn, const hyena_film_t* film, int B, int N,
                                     int D, int L, float* h, void* stream)
{
    hyena_status_t s = check_ffn(ffn);
    if (s != HYENA_OK) return s;
    if (!film || !h || B < 1 || N < 1 || D < 1 || L < 1 || !aligned(h, 4)) return HYENA_ERR_INVALID_ARG;
    const void* p[4] = {film->omega, film->gamma, film->beta, film->sigma};
    for (const void* q : p)
        if (q && !aligned(q, 4)) return HYENA_ERR_INVALID_ARG;
    if (B > 65535 || (long)N * D > 65535L * kFgRowTile || (long)B * N * D * (long)L > (1L << 40))
        return HYENA_ERR_UNSUPPORTED;
    return filter_gen(ffn, N * D, D, L, L, 0, 0, false, h, (cudaStream_t)stream, film, B);
}

hyena_status_t hyena_filter_gen_film_2d(const hyena_ffn_t* ffn, const hyena_film_t* film, int B, int N,
                                        int C, int H, int W, float* h, void* stream)
{
    hyena_status_t s = check_ffn(ffn);
    if (s != HYENA_OK) return s;
    if (!film || !h || B < 1 || N < 1 || C < 1 || H < 1 || W < 1 || !aligned(h, 4))
        return HYENA_ERR_INVALID_ARG;
    const void* p[4] = {film->omega, film->gamma, film->beta, film->sigma};
    for (const void* q : p)
        if (q && !aligned(q, 4)) return HYENA_ERR_INVALID_ARG;
    if (B > 65535 || (long)H * W > (1L << 30) || (long)N * C > 65535L * kFgRowTile ||
        (long)B * N * C * (long)H * W > (1L << 40))
        return HYENA_ERR_UNSUPPORTED;
    return filter_gen(ffn, N * C, C, (long)H * W, 0, H, W, true, h, (cudaStream_t)stream, film, B);
}

hyena_status_t hyena_filter_gen_2d(const hyena_ffn_t* ffn, int N, int C, int H, int W, float* h,
                                   void* stream)
{
    hyena_status_t s = check_ffn(ffn);
    if (s != HYENA_OK) return s;
    if (!h || N < 1 || C < 1 || H < 1 || W < 1 || !aligned(h, 4)) return HYENA_ERR_INVALID_ARG;
    if ((long)H * W > (1L << 30) || (long)N * C > 65535L * kFgRowTile ||
        (long)N * C * (long)H * W > (1L << 40))
        return HYENA_ERR_UNSUPPORTED;
    return filter_gen(ffn, N * C, C, (long)H * W, 0, H, W, true, h, (cudaStream_t)stream);
}

hyena_status_t hyena_filter_gen_3d(const hyena_ffn_t* ffn, int N, int C, int Z, int H, int W, float* h,
                                   void* stream)
{
    hyena_status_t s = check_ffn(ffn);
    if (s != HYENA_OK) return s;
    if (!h || N < 1 || C < 1 || Z < 1 || H < 1 || W < 1 || !aligned(h, 4)) return HYENA_ERR_INVALID_ARG;
    if (ffn->n_bands > kFg3dBands) return HYENA_ERR_UNSUPPORTED;
    const long npos = (long)Z * H * W;
    if (npos > (1L << 30) || (long)N * C > 65535L * kFgRowTile || (long)N * C * npos > (1L << 40))
        return HYENA_ERR_UNSUPPORTED;
    return filter_gen(ffn, N * C, C, npos, 0, H, W, true, h, (cudaStream_t)stream, nullptr, 1, Z);
}

hyena_status_t hyena_filter_gen_film_3d(const hyena_ffn_t* ffn, const hyena_film_t* film, int B, int N,
                                        int C, int Z, int H, int W, float* h, void* stream)
{
    hyena_status_t s = check_ffn(ffn);
    if (s != HYENA_OK) return s;
    if (!film || !h || B < 1 || N < 1 || C < 1 || Z < 1 || H < 1 || W < 1 || !aligned(h, 4))
        return HYENA_ERR_INVALID_ARG;
    const void* p[4] = {film->omega, film->gamma, film->beta, film->sigma};
    for (const void* q : p)
        if (q && !aligned(q, 4)) return HYENA_ERR_INVALID_ARG;
    if (ffn->n_bands > kFg3dBands) return HYENA_ERR_UNSUPPORTED;
    const long npos = (long)Z * H * W;
    if (B > 65535 || npos > (1L << 30) || (long)N * C > 65535L * kFgRowTile ||
        (long)B * N * C * npos > (1L << 40))
        return HYENA_ERR_UNSUPPORTED;
    return filter_gen(ffn, N * C, C, npos, 0, H, W, true, h, (cudaStream_t)stream, film, B, Z);
}

size_t hyena_filter_rfft_workspace_size(int N, int D, int L)
{
    int log2m = 0;
    if (N < 1 || D < 1 || check_len(L, kMaxLog2, &log2m) != HYENA_OK) return (size_t)-1;
    return log2m <= kMaxLog2Fused ? 0 : round_up(scratch_bytes((long)N * D, L), 256);
}

hyena_status_t hyena_filter_rfft(const float* h, int N, int D, int L, float* H, void* workspace,
                                 size_t ws_bytes, void* stream)
{
    if (!h || !H || N < 1 || D < 1) return HYENA_ERR_INVALID_ARG;
    int log2m = 0;
    hyena_status_t s = check_len(L, kMaxLog2, &log2m);
    if (s != HYENA_OK) return s;
    if (!aligned(h, 16) || !aligned(H, 16)) return HYENA_ERR_INVALID_ARG;
    if ((long)N * D > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    const size_t spec = spectrum_bytes(N, D, L);
    if (overlap(h, sizeof(float) * N * D * (size_t)L, H, spec)) return HYENA_ERR_INVALID_ARG;
    const size_t need = log2m <= kMaxLog2Fused ? 0 : round_up(scratch_bytes((long)N * D, L), 256);
    if (need > 0) {
        if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return HYENA_ERR_WORKSPACE;
        if (overlap(workspace, need, H, spec) || overlap(workspace, need, h, sizeof(float) * N * D * (size_t)L))
            return HYENA_ERR_INVALID_ARG;
    }
    return spectra(log2m, h, N * D, reinterpret_cast<float2*>(H), reinterpret_cast<float2*>(workspace),
                   (cudaStream_t)stream);
}

size_t hyena_fftconv_workspace_size(int B, int D, int L, int N, hyena_dtype_t io,
                                    int spectrum_given)
{
    int log2m = 0;
    if (B < 1 || D < 1 || N < 1 || N > HYENA_MAX_ORDER || (io != HYENA_F32 && io != HYENA_BF16))
        return (size_t)-1;
    if (check_len(L, kMaxLog2, &log2m) != HYENA_OK) return (size_t)-1;
    size_t need = spectrum_given ? 0 : round_up(spectrum_bytes(N, D, L), 256);
    if (log2m > kMaxLog2Fused) {
        const long nseq = (long)B * D > (long)N * D ? (long)B * D : (long)N * D;
        need += round_up(scratch_bytes(nseq, L), 256);
    }
    return need;
}

hyena_status_t hyena_fftconv_gate_forward(const void* v, const void* const* x, const float* h,
                                          const float* H, const float* bias, int B, int D, int L,
                                          int N, hyena_dtype_t io, void* y, void* workspace,
                                          size_t ws_bytes, void* stream)
{
    return forward_impl(v, x, h, H, false, bias, B, D, L, N, io, y, workspace, ws_bytes, stream);
}

hyena_status_t hyena_fftconv_gate_forward_per_sample(const void* v, const void* const* x,
                                                     const float* H, const float* bias, int B, int D,
                                                     int L, int N, hyena_dtype_t io, void* y,
                                                     void* workspace, size_t ws_bytes, void* stream)
{
    if (!H) return HYENA_ERR_INVALID_ARG;
    return forward_impl(v, x, nullptr, H, true, bias, B, D, L, N, io, y, workspace, ws_bytes, stream);
}

}  // extern "C"

namespace {

// The forward; per_sample: H holds B spectrum sets [B][N][D][L].
hyena_status_t forward_impl(const void* v, const void* const* x, const float* h, const float* H,
                            bool per_sample, const float* bias, int B, int D, int L, int N,
                            hyena_dtype_t io, void* y, void* workspace, size_t ws_bytes, void* stream)
{
    if (!v || !x || !y || !bias || (!h && !H)) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || D < 1 || N < 1 || L < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_ORDER) return HYENA_ERR_UNSUPPORTED;
    int log2m = 0;
    hyena_status_t s = check_len(L, kMaxLog2, &log2m);
    if (s != HYENA_OK) return s;
    if ((long)B * D > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !aligned(x[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!aligned(v, 16) || !aligned(y, 16) || !aligned(bias, 4)) return HYENA_ERR_INVALID_ARG;
    if ((H && !aligned(H, 16)) || (!H && !aligned(h, 16))) return HYENA_ERR_INVALID_ARG;

    const size_t act = (size_t)B * D * L * io_bytes(io);
    const size_t spec = spectrum_bytes(N, D, L) * (per_sample ? (size_t)B : 1);
    const size_t need = hyena_fftconv_workspace_size(B, D, L, N, io, H != nullptr);
    if (need > 0 && (!workspace || ws_bytes < need || !aligned(workspace, 256)))
        return HYENA_ERR_WORKSPACE;
    // y must not overlap anything it is computed from
    if (overlap(y, act, v, act) || overlap(y, act, bias, sizeof(float) * N * D) ||
        (H && overlap(y, act, H, spec)) ||
        (!H && overlap(y, act, h, sizeof(float) * N * D * (size_t)L)) ||
        (need > 0 && overlap(y, act, workspace, need)))
        return HYENA_ERR_INVALID_ARG;
    for (int n = 0; n < N; ++n)
        if (overlap(y, act, x[n], act) || (need > 0 && overlap(workspace, need, x[n], act)))
            return HYENA_ERR_INVALID_ARG;
    if (need > 0 && (overlap(workspace, need, v, act) || (H && overlap(workspace, need, H, spec)) ||
                     (!H && overlap(h, sizeof(float) * N * D * (size_t)L, workspace, need))))
        return HYENA_ERR_INVALID_ARG;

    cudaStream_t st = (cudaStream_t)stream;
    char* ws = static_cast<char*>(workspace);
    const float2* spectrum = reinterpret_cast<const float2*>(H);
    float2* scratch = nullptr;
    if (!H) {
        float2* Hw = reinterpret_cast<float2*>(ws);
        ws += round_up(spec, 256);
        if (log2m > kMaxLog2Fused) scratch = reinterpret_cast<float2*>(ws);
        s = spectra(log2m, h, N * D, Hw, scratch, st);
        if (s != HYENA_OK) return s;
        spectrum = Hw;
    } else if (log2m > kMaxLog2Fused) {
        scratch = reinterpret_cast<float2*>(ws);
    }
    if (log2m <= kMaxLog2Fused) {
        Fused1dArgs a = {};
        a.v = v;
        for (int n = 0; n < kMaxOrder; ++n) a.x[n] = n < N ? x[n] : nullptr;
        a.y = y;
        a.H = spectrum;
        a.bias = bias;
        a.B = B;
        a.D = D;
        a.N = N;
        a.H_bstride = per_sample ? (size_t)N * D * L : 0;
        return io == HYENA_BF16 ? dispatch_fused_bf16(log2m, a, st) : dispatch_fused_f32(log2m, a, st);
    }
    FourStepArgs a = {};
    a.v = v;
    for (int n = 0; n < kMaxOrder; ++n) a.x[n] = n < N ? x[n] : nullptr;
    a.y = y;
    a.H = spectrum;
    a.H_bstride = per_sample ? (size_t)N * D * L : 0;
    a.bias = bias;
    a.B = B;
    a.D = D;
    return io == HYENA_BF16 ? dispatch_fourstep_bf16(log2m, a, N, scratch, st)
                            : dispatch_fourstep_f32(log2m, a, N, scratch, st);
}

}  // namespace

extern "C" {

size_t hyena_filter_rfft_circular_workspace_size(int N, int D, int L)
{
    const int k = exact_log2(L);
    if (N < 1 || D < 1 || k < kMinLog2Circ + 1 || k > kMaxLog2) return (size_t)-1;
    return k - 1 <= kMaxLog2Circ ? 0 : round_up(scratch_bytes((long)N * D, L / 2), 256);
}

hyena_status_t hyena_filter_rfft_circular(const float* h, int N, int D, int L, float* H, void* workspace,
                                          size_t ws_bytes, void* stream)
{
    if (!h || !H || N < 1 || D < 1 || L < 1) return HYENA_ERR_INVALID_ARG;
    const int k = exact_log2(L);
    if (k < kMinLog2Circ + 1 || k > kMaxLog2) return HYENA_ERR_UNSUPPORTED;
    if (!aligned(h, 16) || !aligned(H, 16)) return HYENA_ERR_INVALID_ARG;
    if ((long)N * D > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    const size_t spec = sizeof(float2) * (size_t)N * D * (L / 2);
    if (overlap(h, sizeof(float) * (size_t)N * D * L, H, spec)) return HYENA_ERR_INVALID_ARG;
    if (k - 1 > kMaxLog2Circ) {
        // four-step (L > 16384): a wave of rows through the workspace
        const size_t need = hyena_filter_rfft_circular_workspace_size(N, D, L);
        if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return HYENA_ERR_WORKSPACE;
        if (overlap(workspace, need, h, sizeof(float) * (size_t)N * D * L) || overlap(workspace, need, H, spec))
            return HYENA_ERR_INVALID_ARG;
        return dispatch_fourstep_rfft_circ(k - 1, h, N * D, reinterpret_cast<float2*>(H),
                                           static_cast<float2*>(workspace), (cudaStream_t)stream);
    }
    Rfft1dArgs ra;
    ra.h = h;
    ra.H = reinterpret_cast<float2*>(H);
    ra.rows = N * D;
    return dispatch_rfft_circ(k - 1, ra, (cudaStream_t)stream);
}

size_t hyena_fftconv_circular_workspace_size(int B, int D, int L, int N)
{
    const int k = exact_log2(L);
    if (B < 1 || D < 1 || N < 1 || N > HYENA_MAX_ORDER || k < kMinLog2Circ + 1 || k > kMaxLog2)
        return (size_t)-1;
    return k - 1 <= kMaxLog2Circ ? 0 : round_up(scratch_bytes((long)B * D, L / 2), 256);
}

static hyena_status_t hyena_fftconv_gate_forward_circular_impl(bool per_sample, const void* v, const void* const* x, const float* H,
                                                   const float* bias, int B, int D, int L, int N,
                                                   hyena_dtype_t io, void* y, void* workspace, size_t ws_bytes,
                                                   void* stream)
{
    if (!v || !x || !H || !bias || !y) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || D < 1 || N < 1 || L < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_ORDER || (long)B * D > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    const int k = exact_log2(L);
    if (k < kMinLog2Circ + 1 || k > kMaxLog2) return HYENA_ERR_UNSUPPORTED;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !aligned(x[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!aligned(v, 16) || !aligned(y, 16) || !aligned(H, 16) || !aligned(bias, 4))
        return HYENA_ERR_INVALID_ARG;
    const size_t act = (size_t)B * D * L * io_bytes(io);
    const size_t spec = sizeof(float2) * (size_t)N * D * (L / 2) * (per_sample ? (size_t)B : 1);
    if (overlap(y, act, v, act) || overlap(y, act, H, spec) || overlap(y, act, bias, sizeof(float) * N * D))
        return HYENA_ERR_INVALID_ARG;
    for (int n = 0; n < N; ++n)
        if (overlap(y, act, x[n], act)) return HYENA_ERR_INVALID_ARG;
    const size_t need = hyena_fftconv_circular_workspace_size(B, D, L, N);
    if (need > 0) {
        if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return HYENA_ERR_WORKSPACE;
        if (overlap(y, act, workspace, need) || overlap(workspace, need, v, act) ||
            overlap(workspace, need, H, spec))
            return HYENA_ERR_INVALID_ARG;
        for (int n = 0; n < N; ++n)
            if (overlap(workspace, need, x[n], act)) return HYENA_ERR_INVALID_ARG;
    }
    cudaStream_t st = (cudaStream_t)stream;
    if (k - 1 > kMaxLog2Circ) {
        // four-step (L > 16384)
        FourStepArgs a = {};
        a.v = v;
        for (int n = 0; n < kMaxOrder; ++n) a.x[n] = n < N ? x[n] : nullptr;
        a.y = y;
        a.H = reinterpret_cast<const float2*>(H);
        a.H_bstride = per_sample ? (size_t)N * D * (L / 2) : 0;
        a.bias = bias;
        a.B = B;
        a.D = D;
        float2* scratch = static_cast<float2*>(workspace);
        return io == HYENA_BF16 ? dispatch_fourstep_circ_bf16(k - 1, a, N, scratch, st)
                                : dispatch_fourstep_circ_f32(k - 1, a, N, scratch, st);
    }
    Fused1dArgs a = {};
    a.v = v;
    for (int n = 0; n < kMaxOrder; ++n) a.x[n] = n < N ? x[n] : nullptr;
    a.y = y;
    a.H = reinterpret_cast<const float2*>(H);
    a.H_bstride = per_sample ? (size_t)N * D * (L / 2) : 0;
    a.bias = bias;
    a.B = B;
    a.D = D;
    a.N = N;
    if (per_sample)
        return io == HYENA_BF16 ? dispatch_fused_circ_ps_bf16(k - 1, a, st) : dispatch_fused_circ_ps_f32(k - 1, a, st);
    return io == HYENA_BF16 ? dispatch_fused_circ_bf16(k - 1, a, st) : dispatch_fused_circ_f32(k - 1, a, st);
}

hyena_status_t hyena_fftconv_gate_forward_circular(const void* v, const void* const* x, const float* H,
                                                   const float* bias, int B, int D, int L, int N,
                                                   hyena_dtype_t io, void* y, void* workspace, size_t ws_bytes,
                                                   void* stream)
{
    return hyena_fftconv_gate_forward_circular_impl(false, v, x, H, bias, B, D, L, N, io, y, workspace, ws_bytes, stream);
}

hyena_status_t hyena_fftconv_gate_forward_circular_per_sample(const void* v, const void* const* x, const float* H,
                                                   const float* bias, int B, int D, int L, int N,
                                                   hyena_dtype_t io, void* y, void* workspace, size_t ws_bytes,
                                                   void* stream)
{
    return hyena_fftconv_gate_forward_circular_impl(true, v, x, H, bias, B, D, L, N, io, y, workspace, ws_bytes, stream);
}


size_t hyena_fftconv_backward_workspace_size(int B, int D, int L, int N)
{
    int log2m = 0;
    if (B < 1 || D < 1 || N < 1 || N > HYENA_MAX_ORDER || check_len(L, kMaxLog2, &log2m) != HYENA_OK)
        return (size_t)-1;
    if (log2m > kMaxLog2Fused) return fourstep_bwd_layout(log2m, D, N).total;
    return bwd1d_layout(B, D, L, N, false, false).total;
}

size_t hyena_fftconv_backward_per_sample_workspace_size(int B, int D, int L, int N)
{
    int log2m = 0;
    if (B < 1 || D < 1 || N < 1 || N > HYENA_MAX_ORDER || check_len(L, kMaxLog2, &log2m) != HYENA_OK)
        return (size_t)-1;
    if (log2m > kMaxLog2Fused) return fourstep_bwd_layout(log2m, D, N, B).total;
    return bwd1d_layout(B, D, L, N, true, false).total;
}

hyena_status_t hyena_fftconv_gate_backward(const void* v, const void* const* x, const float* H,
                                           const float* bias, const void* dy, int B, int D, int L,
                                           int N, hyena_dtype_t io, void* dv, void* const* dx,
                                           float* dh, float* dbias, void* workspace, size_t ws_bytes,
                                           void* stream)
{
    return backward_impl(v, x, H, false, false, bias, dy, B, D, L, N, io, dv, dx, dh, dbias, workspace,
                         ws_bytes, stream);
}

size_t hyena_fftconv_backward_circular_workspace_size(int B, int D, int L, int N)
{
    const int k = exact_log2(L);
    if (B < 1 || D < 1 || N < 1 || N > HYENA_MAX_ORDER || k < kMinLog2Circ + 1 || k > kMaxLog2)
        return (size_t)-1;
    if (k - 1 > kMaxLog2Circ) return fourstep_bwd_layout(k - 1, D, N, 1, true).total;   // four-step
    return bwd1d_layout(B, D, L, N, false, true).total;
}

hyena_status_t hyena_fftconv_gate_backward_circular(const void* v, const void* const* x, const float* H,
                                                    const float* bias, const void* dy, int B, int D, int L,
                                                    int N, hyena_dtype_t io, void* dv, void* const* dx,
                                                    float* dh, float* dbias, void* workspace,
                                                    size_t ws_bytes, void* stream)
{
    return backward_impl(v, x, H, false, true, bias, dy, B, D, L, N, io, dv, dx, dh, dbias, workspace,
                         ws_bytes, stream);
}

size_t hyena_fftconv_backward_circular_per_sample_workspace_size(int B, int D, int L, int N)
{
    const int k = exact_log2(L);
    if (B < 1 || D < 1 || N < 1 || N > HYENA_MAX_ORDER || k < kMinLog2Circ + 1 || k > kMaxLog2) return (size_t)-1;
    if (k - 1 > kMaxLog2Circ) return fourstep_bwd_layout(k - 1, D, N, B, true).total;   // four-step
    return bwd1d_layout(B, D, L, N, true, true).total;
}

hyena_status_t hyena_fftconv_gate_backward_circular_per_sample(const void* v, const void* const* x,
                                                               const float* H, const float* bias, const void* dy,
                                                               int B, int D, int L, int N, hyena_dtype_t io,
                                                               void* dv, void* const* dx, float* dh, float* dbias,
                                                               void* workspace, size_t ws_bytes, void* stream)
{
    return backward_impl(v, x, H, true, true, bias, dy, B, D, L, N, io, dv, dx, dh, dbias, workspace,
                         ws_bytes, stream);
}

hyena_status_t hyena_fftconv_gate_backward_per_sample(const void* v, const void* const* x, const float* H,
                                                      const float* bias, const void* dy, int B, int D, int L,
                                                      int N, hyena_dtype_t io, void* dv, void* const* dx,
                                                      float* dh, float* dbias, void* workspace,
                                                      size_t ws_bytes, void* stream)
{
    return backward_impl(v, x, H, true, false, bias, dy, B, D, L, N, io, dv, dx, dh, dbias, workspace,
                         ws_bytes, stream);
}

}  // extern "C"

namespace {

// per_sample: a spectrum set per sample (L <= 16384); circular: the
// circular recurrence (32 <= L <= 16384, spectra of L/2 slots)
hyena_status_t backward_impl(const void* v, const void* const* x, const float* H, bool per_sample,
                             bool circular, const float* bias, const void* dy, int B, int D, int L, int N,
                             hyena_dtype_t io, void* dv, void* const* dx, float* dh, float* dbias,
                             void* workspace, size_t ws_bytes, void* stream)
{
    if (!v || !x || !H || !bias || !dy || !dv || !dx || !dh || !dbias) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || D < 1 || N < 1 || L < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_ORDER) return HYENA_ERR_UNSUPPORTED;
    int log2m = 0;
    if (circular) {
        const int k = exact_log2(L);
        if (k < kMinLog2Circ + 1 || k > kMaxLog2) return HYENA_ERR_UNSUPPORTED;
        log2m = k - 1;                       // M = L/2 packed points
    } else {
        hyena_status_t s = check_len(L, kMaxLog2, &log2m);
        if (s != HYENA_OK) return s;
    }
    if ((long)B * D > (1L << 30) || (per_sample && (long)B * N * D > (1L << 30))) return HYENA_ERR_UNSUPPORTED;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !dx[n] || !aligned(x[n], 16) || !aligned(dx[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!aligned(v, 16) || !aligned(dy, 16) || !aligned(dv, 16) || !aligned(H, 16) || !aligned(dh, 16) ||
        !aligned(bias, 4) || !aligned(dbias, 4))
        return HYENA_ERR_INVALID_ARG;
    const size_t need = circular ? (per_sample ? hyena_fftconv_backward_circular_per_sample_workspace_size(B, D, L, N)
                                               : hyena_fftconv_backward_circular_workspace_size(B, D, L, N))
                        : per_sample ? hyena_fftconv_backward_per_sample_workspace_size(B, D, L, N)
                                     : hyena_fftconv_backward_workspace_size(B, D, L, N);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return HYENA_ERR_WORKSPACE;
    const size_t sets = per_sample ? (size_t)B : 1;           // spectrum sets and dh sets

    // every output against every input, the other outputs and the workspace
    const size_t act = (size_t)B * D * L * io_bytes(io);
    struct Range { const void* p; size_t n; };
    Range in[kMaxOrder + 5], out[kMaxOrder + 3];
    int ni = 0, no = 0;
    in[ni++] = {v, act};
    in[ni++] = {dy, act};
    in[ni++] = {H, spectrum_bytes(N, D, circular ? L / 2 : L) * sets};
    in[ni++] = {bias, sizeof(float) * N * D};
    in[ni++] = {workspace, need};
    for (int n = 0; n < N; ++n) in[ni++] = {x[n], act};
    out[no++] = {dv, act};
    out[no++] = {dh, sizeof(float) * (size_t)N * D * L * sets};
    out[no++] = {dbias, sizeof(float) * N * D};
    for (int n = 0; n < N; ++n) out[no++] = {dx[n], act};
    for (int o = 0; o < no; ++o) {
        for (int i = 0; i < ni; ++i)
            if (overlap(out[o].p, out[o].n, in[i].p, in[i].n)) return HYENA_ERR_INVALID_ARG;
        for (int p = o + 1; p < no; ++p)
            if (overlap(out[o].p, out[o].n, out[p].p, out[p].n)) return HYENA_ERR_INVALID_ARG;
    }

    char* ws = static_cast<char*>(workspace);
    cudaStream_t st = (cudaStream_t)stream;
    if (circular ? log2m > kMaxLog2Circ : log2m > kMaxLog2Fused) {
        // four-step backward (L > 16384)
        const FourStepBwdLayout lay = fourstep_bwd_layout(log2m, D, N, (int)sets, circular);
        FourStepBwdArgs b = {};
        b.f.v = v;
        for (int n = 0; n < kMaxOrder; ++n) {
            b.f.x[n] = n < N ? x[n] : nullptr;
            b.dx[n] = n < N ? dx[n] : nullptr;
        }
        b.f.H = reinterpret_cast<const float2*>(H);
        b.f.H_bstride = per_sample ? (size_t)N * D * (circular ? L / 2 : L) : 0;
        b.f.bias = bias;
        b.f.S = reinterpret_cast<float2*>(ws + lay.scratch);
        b.f.B = B;
        b.f.D = D;
        b.dy = dy;
        b.dv = dv;
        b.zsave = reinterpret_cast<float2*>(ws + lay.zsave);
        b.csave = reinterpret_cast<float2*>(ws + lay.csave);
        b.acc = reinterpret_cast<float2*>(ws + lay.acc);
        b.dh = dh;
        b.dbias = dbias;
        b.wcap = (int)lay.wcap;
        if (circular)
            return io == HYENA_BF16 ? dispatch_fourstep_bwd_circ_bf16(log2m, b, N, st)
                                    : dispatch_fourstep_bwd_circ_f32(log2m, b, N, st);
        return io == HYENA_BF16 ? dispatch_fourstep_bwd_bf16(log2m, b, N, st)
                                : dispatch_fourstep_bwd_f32(log2m, b, N, st);
    }
    Backward1dArgs a;
    a.v = v;
    a.dy = dy;
    for (int n = 0; n < kMaxOrder; ++n) {
        a.x[n] = n < N ? x[n] : nullptr;
        a.dx[n] = n < N ? dx[n] : nullptr;
    }
    a.H = reinterpret_cast<const float2*>(H);
    a.bias = bias;
    a.dv = dv;
    a.dh = dh;
    a.dbias = dbias;
    const Bwd1dLayout lay = bwd1d_layout(B, D, L, N, per_sample, circular);
    a.acc = reinterpret_cast<float2*>(ws + lay.acc);
    a.wz = reinterpret_cast<float2*>(ws + lay.wz);
    a.wc = reinterpret_cast<float2*>(ws + lay.wc);
    a.B = B;
    a.D = D;
    a.N = N;
    a.S = lay.slices;                        // the most batch slices the workspace holds
    a.H_bstride = per_sample ? (size_t)N * D * (circular ? L / 2 : L) : 0;
    if (circular && per_sample)
        return io == HYENA_BF16 ? dispatch_backward_circ_ps_bf16(log2m, a, st)
                                : dispatch_backward_circ_ps_f32(log2m, a, st);
    if (circular)
        return io == HYENA_BF16 ? dispatch_backward_circ_bf16(log2m, a, st)
                                : dispatch_backward_circ_f32(log2m, a, st);
    if (per_sample)
        return io == HYENA_BF16 ? dispatch_backward_ps_bf16(log2m, a, st) : dispatch_backward_ps_f32(log2m, a, st);
    return io == HYENA_BF16 ? dispatch_backward_bf16(log2m, a, st) : dispatch_backward_f32(log2m, a, st);
}

}  // namespace

extern "C" {

// ------------------------------------------------------------------ 2-D

size_t hyena_fftconv2d_workspace_size(int B, int C, int H, int W, int N, hyena_dtype_t io,
                                      int spectrum_given)
{
    if (B < 1 || C < 1 || N < 1 || N > HYENA_MAX_ORDER || (io != HYENA_F32 && io != HYENA_BF16))
        return (size_t)-1;
    const int lh = exact_log2(H), lw = exact_log2(W);
    if (lh < kMinLog2H2d || lh > kMaxLog2H2d || lw < kMinLog2W2d || lw > kMaxLog2W2d) return (size_t)-1;
    size_t need = spectrum_given ? 0 : round_up(sizeof(float2) * (size_t)N * C * 2 * H * W, 256);
    return need + round_up(sizeof(float2) * (size_t)wave_images((long)B * C, H, W) * H * W, 256);
}

hyena_status_t hyena_filter_rfft2d(const float* h, int N, int C, int H, int W, float* Hs, void* stream)
{
    if (!h || !Hs || N < 1 || C < 1 || H < 1 || W < 1) return HYENA_ERR_INVALID_ARG;
    const int lh = exact_log2(H), lw = exact_log2(W);
    if (lh < kMinLog2H2d || lh > kMaxLog2H2d || lw < kMinLog2W2d || lw > kMaxLog2W2d)
        return HYENA_ERR_UNSUPPORTED;
    if ((long)N * C > (1L << 20)) return HYENA_ERR_UNSUPPORTED;
    if (!aligned(h, 16) || !aligned(Hs, 16)) return HYENA_ERR_INVALID_ARG;
    if (overlap(h, sizeof(float) * (size_t)N * C * H * W, Hs, sizeof(float2) * (size_t)N * C * 2 * H * W))
        return HYENA_ERR_INVALID_ARG;
    Fft2dArgs a = {};
    a.v = h;
    a.S = reinterpret_cast<float2*>(Hs);
    a.B = 1;
    a.C = N * C;
    a.H = H;
    a.W = W;
    a.nq = N * C;
    return dispatch_rfft2d(lw, lh, a, (cudaStream_t)stream);
}

hyena_status_t hyena_fftconv2d_gate_forward(const void* v, const void* const* x, const float* h,
                                            const float* Hs, const float* bias, int B, int C, int H,
                                            int W, int N, hyena_dtype_t io, void* y, void* workspace,
                                            size_t ws_bytes, void* stream)
{
    return forward2d_impl(v, x, h, Hs, false, bias, B, C, H, W, N, io, y, workspace, ws_bytes, stream);
}

hyena_status_t hyena_fftconv2d_gate_forward_per_sample(const void* v, const void* const* x, const float* Hs,
                                                       const float* bias, int B, int C, int H, int W, int N,
                                                       hyena_dtype_t io, void* y, void* workspace,
                                                       size_t ws_bytes, void* stream)
{
    if (!Hs) return HYENA_ERR_INVALID_ARG;
    return forward2d_impl(v, x, nullptr, Hs, true, bias, B, C, H, W, N, io, y, workspace, ws_bytes, stream);
}

}  // extern "C"

namespace {

hyena_status_t forward2d_impl(const void* v, const void* const* x, const float* h, const float* Hs,
                              bool per_sample, const float* bias, int B, int C, int H, int W, int N,
                              hyena_dtype_t io, void* y, void* workspace, size_t ws_bytes, void* stream)
{
    if (!v || !x || !y || !bias || (!h && !Hs)) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || C < 1 || N < 1 || H < 1 || W < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_ORDER) return HYENA_ERR_UNSUPPORTED;
    const int lh = exact_log2(H), lw = exact_log2(W);
    if (lh < kMinLog2H2d || lh > kMaxLog2H2d || lw < kMinLog2W2d || lw > kMaxLog2W2d)
        return HYENA_ERR_UNSUPPORTED;
    if ((long)B * C > (1L << 20) || (long)N * C > (1L << 20)) return HYENA_ERR_UNSUPPORTED;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !aligned(x[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!aligned(v, 16) || !aligned(y, 16) || !aligned(bias, 4)) return HYENA_ERR_INVALID_ARG;
    if ((Hs && !aligned(Hs, 16)) || (!Hs && !aligned(h, 16))) return HYENA_ERR_INVALID_ARG;

    const size_t act = (size_t)B * C * H * W * io_bytes(io);
    const size_t spec = sizeof(float2) * (size_t)N * C * 2 * H * W * (per_sample ? (size_t)B : 1);
    const size_t filt = sizeof(float) * (size_t)N * C * H * W;
    const size_t need = hyena_fftconv2d_workspace_size(B, C, H, W, N, io, Hs != nullptr);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return HYENA_ERR_WORKSPACE;
    if (overlap(y, act, v, act) || overlap(y, act, bias, sizeof(float) * N * C) ||
        (Hs && overlap(y, act, Hs, spec)) || (!Hs && overlap(y, act, h, filt)) ||
        overlap(y, act, workspace, need) || overlap(workspace, need, v, act) ||
        (Hs && overlap(workspace, need, Hs, spec)) || (!Hs && overlap(workspace, need, h, filt)))
        return HYENA_ERR_INVALID_ARG;
    for (int n = 0; n < N; ++n)
        if (overlap(y, act, x[n], act) || overlap(workspace, need, x[n], act))
            return HYENA_ERR_INVALID_ARG;

    cudaStream_t st = (cudaStream_t)stream;
    char* ws = static_cast<char*>(workspace);
    const float2* spectrum = reinterpret_cast<const float2*>(Hs);
    if (!Hs) {
        Fft2dArgs sa = {};
        sa.v = h;
        sa.S = reinterpret_cast<float2*>(ws);
        sa.B = 1;
        sa.C = N * C;
        sa.H = H;
        sa.W = W;
        sa.nq = N * C;
        hyena_status_t s = dispatch_rfft2d(lw, lh, sa, st);
        if (s != HYENA_OK) return s;
        spectrum = sa.S;
        ws += round_up(spec, 256);
    }
    Fft2dArgs a = {};
    a.v = v;
    for (int n = 0; n < kMaxOrder; ++n) a.x[n] = n < N ? x[n] : nullptr;
    a.y = y;
    a.Hs = spectrum;
    a.Hs_bstride = per_sample ? (size_t)N * C * 2 * H * W : 0;
    a.bias = bias;
    a.B = B;
    a.C = C;
    a.H = H;
    a.W = W;
    float2* scratch = reinterpret_cast<float2*>(ws);
    return io == HYENA_BF16 ? dispatch_fft2d_bf16(lw, lh, a, N, scratch, st)
                            : dispatch_fft2d_f32(lw, lh, a, N, scratch, st);
}

}  // namespace

extern "C" {

}  // extern "C"

namespace {

bool dims3d_ok(int Z, int H, int W, int& lz, int& lh, int& lw)
{
    lz = exact_log2(Z);
    lh = exact_log2(H);
    lw = exact_log2(W);
    return lz >= kMinLog2_3d && lz <= kMaxLog2_3d && lh >= kMinLog2_3d && lh <= kMaxLog2_3d &&
           lw >= kMinLog2_3d && lw <= kMaxLog2_3d;
}

}  // namespace

extern "C" {

size_t hyena_fftconv3d_workspace_size(int B, int C, int Z, int H, int W, int N, hyena_dtype_t io,
                                      int spectrum_given)
{
    if (B < 1 || C < 1 || N < 1 || N > HYENA_MAX_ORDER || (io != HYENA_F32 && io != HYENA_BF16))
        return (size_t)-1;
    int lz, lh, lw;
    if (!dims3d_ok(Z, H, W, lz, lh, lw)) return (size_t)-1;
    const size_t vol2 = (size_t)Z * 2 * H * W;                  // slots of one scratch volume
    size_t need = spectrum_given ? 0 : round_up(sizeof(float2) * (size_t)N * C * 2 * vol2, 256);
    return need + round_up(sizeof(float2) * (size_t)wave_images_3d((long)B * C, Z, H, W) * vol2, 256);
}

hyena_status_t hyena_filter_rfft3d(const float* h, int N, int C, int Z, int H, int W, float* Hs, void* stream)
{
    if (!h || !Hs || N < 1 || C < 1 || Z < 1 || H < 1 || W < 1) return HYENA_ERR_INVALID_ARG;
    int lz, lh, lw;
    if (!dims3d_ok(Z, H, W, lz, lh, lw)) return HYENA_ERR_UNSUPPORTED;
    if ((long)N * C * Z * H > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    if (!aligned(h, 16) || !aligned(Hs, 16)) return HYENA_ERR_INVALID_ARG;
    if (overlap(h, sizeof(float) * (size_t)N * C * Z * H * W, Hs,
                sizeof(float2) * (size_t)N * C * 4 * Z * H * W))
        return HYENA_ERR_INVALID_ARG;
    Fft2dArgs a = {};
    a.v = h;
    a.S = reinterpret_cast<float2*>(Hs);
    a.B = 1;
    a.C = N * C;
    a.W = W;
    a.nq = N * C;
    a.zp = Z;
    a.Hp = H;
    return dispatch_rfft3d(lw, lh, lz, a, (cudaStream_t)stream);
}

hyena_status_t hyena_fftconv3d_gate_forward(const void* v, const void* const* x, const float* h,
                                            const float* Hs, const float* bias, int B, int C, int Z,
                                            int H, int W, int N, hyena_dtype_t io, void* y,
                                            void* workspace, size_t ws_bytes, void* stream)
{
    return forward3d_impl(v, x, h, Hs, false, bias, B, C, Z, H, W, N, io, y, workspace, ws_bytes, stream);
}

hyena_status_t hyena_fftconv3d_gate_forward_per_sample(const void* v, const void* const* x, const float* Hs,
                                                       const float* bias, int B, int C, int Z, int H, int W,
                                                       int N, hyena_dtype_t io, void* y, void* workspace,
                                                       size_t ws_bytes, void* stream)
{
    if (!Hs) return HYENA_ERR_INVALID_ARG;
    return forward3d_impl(v, x, nullptr, Hs, true, bias, B, C, Z, H, W, N, io, y, workspace, ws_bytes,
                          stream);
}

}  // extern "C"

namespace {

hyena_status_t forward3d_impl(const void* v, const void* const* x, const float* h, const float* Hs,
                              bool per_sample, const float* bias, int B, int C, int Z, int H, int W,
                              int N, hyena_dtype_t io, void* y, void* workspace, size_t ws_bytes,
                              void* stream)
{
    if (!v || !x || !y || !bias || (!h && !Hs)) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || C < 1 || N < 1 || Z < 1 || H < 1 || W < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_ORDER) return HYENA_ERR_UNSUPPORTED;
    int lz, lh, lw;
    if (!dims3d_ok(Z, H, W, lz, lh, lw)) return HYENA_ERR_UNSUPPORTED;
    if ((long)B * C > (1L << 20) || (long)N * C * Z * H * (per_sample ? B : 1) > (1L << 30))
        return HYENA_ERR_UNSUPPORTED;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !aligned(x[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!aligned(v, 16) || !aligned(y, 16) || !aligned(bias, 4)) return HYENA_ERR_INVALID_ARG;
    if ((Hs && !aligned(Hs, 16)) || (!Hs && !aligned(h, 16))) return HYENA_ERR_INVALID_ARG;

    const size_t vol = (size_t)Z * H * W;
    const size_t act = (size_t)B * C * vol * io_bytes(io);
    const size_t spec = sizeof(float2) * (size_t)N * C * 4 * vol * (per_sample ? (size_t)B : 1);
    const size_t filt = sizeof(float) * (size_t)N * C * vol;
    const size_t need = hyena_fftconv3d_workspace_size(B, C, Z, H, W, N, io, Hs != nullptr);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return HYENA_ERR_WORKSPACE;
    if (overlap(y, act, v, act) || overlap(y, act, bias, sizeof(float) * N * C) ||
        (Hs && overlap(y, act, Hs, spec)) || (!Hs && overlap(y, act, h, filt)) ||
        overlap(y, act, workspace, need) || overlap(workspace, need, v, act) ||
        (Hs && overlap(workspace, need, Hs, spec)) || (!Hs && overlap(workspace, need, h, filt)))
        return HYENA_ERR_INVALID_ARG;
    for (int n = 0; n < N; ++n)
        if (overlap(y, act, x[n], act) || overlap(workspace, need, x[n], act))
            return HYENA_ERR_INVALID_ARG;

    cudaStream_t st = (cudaStream_t)stream;
    char* ws = static_cast<char*>(workspace);
    const float2* spectrum = reinterpret_cast<const float2*>(Hs);
    if (!Hs) {
        Fft2dArgs sa = {};
        sa.v = h;
        sa.S = reinterpret_cast<float2*>(ws);
        sa.B = 1;
        sa.C = N * C;
        sa.W = W;
        sa.nq = N * C;
        sa.zp = Z;
        sa.Hp = H;
        hyena_status_t s = dispatch_rfft3d(lw, lh, lz, sa, st);
        if (s != HYENA_OK) return s;
        spectrum = sa.S;
        ws += round_up(spec, 256);
    }
    Fft2dArgs a = {};
    a.v = v;
    for (int n = 0; n < kMaxOrder; ++n) a.x[n] = n < N ? x[n] : nullptr;
    a.y = y;
    a.Hs = spectrum;
    a.Hs_bstride = per_sample ? (size_t)N * C * 4 * vol : 0;
    a.bias = bias;
    a.B = B;
    a.C = C;
    a.W = W;
    a.zp = Z;
    a.Hp = H;
    float2* scratch = reinterpret_cast<float2*>(ws);
    return io == HYENA_BF16 ? dispatch_fft3d_bf16(lw, lh, lz, a, N, scratch, st)
                            : dispatch_fft3d_f32(lw, lh, lz, a, N, scratch, st);
}

}  // namespace

// ------------------------------------------------------- circular 2-D

namespace {

// circular 2-D sizes: W in [32, 1024] (rows of W/2 slots), H in [16, 1024]
bool dims2d_circ_ok(int H, int W, int& lh, int& lm)
{
    lh = exact_log2(H);
    const int lw = exact_log2(W);
    lm = lw - 1;
    return lh >= 4 && lh <= 10 && lw >= 5 && lw <= 10;
}

}  // namespace

extern "C" {

size_t hyena_fftconv2d_circular_workspace_size(int B, int C, int H, int W)
{
    int lh, lm;
    if (B < 1 || C < 1 || !dims2d_circ_ok(H, W, lh, lm)) return (size_t)-1;
    return round_up(sizeof(float2) * (size_t)wave_images((long)B * C, H, W / 2) * H * (W / 2), 256);
}

hyena_status_t hyena_filter_rfft2d_circular(const float* h, int N, int C, int H, int W, float* Hs, void* stream)
{
    if (!h || !Hs || N < 1 || C < 1 || H < 1 || W < 1) return HYENA_ERR_INVALID_ARG;
    int lh, lm;
    if (!dims2d_circ_ok(H, W, lh, lm)) return HYENA_ERR_UNSUPPORTED;
    if ((long)N * C > (1L << 20)) return HYENA_ERR_UNSUPPORTED;
    if (!aligned(h, 16) || !aligned(Hs, 16)) return HYENA_ERR_INVALID_ARG;
    if (overlap(h, sizeof(float) * (size_t)N * C * H * W, Hs, sizeof(float2) * (size_t)N * C * H * (W / 2)))
        return HYENA_ERR_INVALID_ARG;
    Fft2dArgs a = {};
    a.v = h;
    a.S = reinterpret_cast<float2*>(Hs);
    a.B = 1;
    a.C = N * C;
    a.H = H;
    a.W = W / 2;
    a.nq = N * C;
    return dispatch_rfft2d_circ(lm, lh, a, (cudaStream_t)stream);
}

static hyena_status_t hyena_fftconv2d_gate_forward_circular_impl(bool per_sample, const void* v, const void* const* x, const float* Hs,
                                                     const float* bias, int B, int C, int H, int W, int N,
                                                     hyena_dtype_t io, void* y, void* workspace,
                                                     size_t ws_bytes, void* stream)
{
    if (!v || !x || !y || !bias || !Hs) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || C < 1 || N < 1 || H < 1 || W < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_ORDER) return HYENA_ERR_UNSUPPORTED;
    int lh, lm;
    if (!dims2d_circ_ok(H, W, lh, lm)) return HYENA_ERR_UNSUPPORTED;
    if ((long)B * C > (1L << 20) || (long)N * C > (1L << 20)) return HYENA_ERR_UNSUPPORTED;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !aligned(x[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!aligned(v, 16) || !aligned(y, 16) || !aligned(bias, 4) || !aligned(Hs, 16)) return HYENA_ERR_INVALID_ARG;
    const size_t act = (size_t)B * C * H * W * io_bytes(io);
    const size_t spec = sizeof(float2) * (size_t)N * C * H * (W / 2) * (per_sample ? (size_t)B : 1);
    const size_t need = hyena_fftconv2d_circular_workspace_size(B, C, H, W);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return HYENA_ERR_WORKSPACE;
    if (overlap(y, act, v, act) || overlap(y, act, bias, sizeof(float) * N * C) || overlap(y, act, Hs, spec) ||
        overlap(y, act, workspace, need) || overlap(workspace, need, v, act) || overlap(workspace, need, Hs, spec))
        return HYENA_ERR_INVALID_ARG;
    for (int n = 0; n < N; ++n)
        if (overlap(y, act, x[n], act) || overlap(workspace, need, x[n], act)) return HYENA_ERR_INVALID_ARG;
    Fft2dArgs a = {};
    a.v = v;
    for (int n = 0; n < kMaxOrder; ++n) a.x[n] = n < N ? x[n] : nullptr;
    a.y = y;
    a.Hs = reinterpret_cast<const float2*>(Hs);
    a.Hs_bstride = per_sample ? (size_t)N * C * H * (W / 2) : 0;
    a.bias = bias;
    a.B = B;
    a.C = C;
    a.H = H;
    a.W = W / 2;
    float2* scratch = static_cast<float2*>(workspace);
    cudaStream_t st = (cudaStream_t)stream;
    return io == HYENA_BF16 ? dispatch_fft2d_circ_bf16(lm, lh, a, N, scratch, st)
                            : dispatch_fft2d_circ_f32(lm, lh, a, N, scratch, st);
}

hyena_status_t hyena_fftconv2d_gate_forward_circular(const void* v, const void* const* x, const float* Hs,
                                                     const float* bias, int B, int C, int H, int W, int N,
                                                     hyena_dtype_t io, void* y, void* workspace,
                                                     size_t ws_bytes, void* stream)
{
    return hyena_fftconv2d_gate_forward_circular_impl(false, v, x, Hs, bias, B, C, H, W, N, io, y, workspace, ws_bytes, stream);
}

hyena_status_t hyena_fftconv2d_gate_forward_circular_per_sample(const void* v, const void* const* x, const float* Hs,
                                                     const float* bias, int B, int C, int H, int W, int N,
                                                     hyena_dtype_t io, void* y, void* workspace,
                                                     size_t ws_bytes, void* stream)
{
    return hyena_fftconv2d_gate_forward_circular_impl(true, v, x, Hs, bias, B, C, H, W, N, io, y, workspace, ws_bytes, stream);
}


}  // extern "C"

// ------------------------------------------------------- circular 3-D

namespace {

// circular 3-D sizes: Z, H in [16, 256], W in [32, 256] (rows of W/2 slots)
bool dims3d_circ_ok(int Z, int H, int W, int& lz, int& lh, int& lm)
{
    lz = exact_log2(Z);
    lh = exact_log2(H);
    const int lw = exact_log2(W);
    lm = lw - 1;
    return lz >= 4 && lz <= 8 && lh >= 4 && lh <= 8 && lw >= 5 && lw <= 8;
}

}  // namespace

extern "C" {

size_t hyena_fftconv3d_circular_workspace_size(int B, int C, int Z, int H, int W)
{
    int lz, lh, lm;
    if (B < 1 || C < 1 || !dims3d_circ_ok(Z, H, W, lz, lh, lm)) return (size_t)-1;
    const size_t vol = (size_t)Z * H * (W / 2);
    return round_up(sizeof(float2) * (size_t)wave_images_3d((long)B * C, Z, H, W / 2, false) * vol, 256);
}

hyena_status_t hyena_filter_rfft3d_circular(const float* h, int N, int C, int Z, int H, int W, float* Hs,
                                            void* stream)
{
    if (!h || !Hs || N < 1 || C < 1 || Z < 1 || H < 1 || W < 1) return HYENA_ERR_INVALID_ARG;
    int lz, lh, lm;
    if (!dims3d_circ_ok(Z, H, W, lz, lh, lm)) return HYENA_ERR_UNSUPPORTED;
    if ((long)N * C * Z * H > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    if (!aligned(h, 16) || !aligned(Hs, 16)) return HYENA_ERR_INVALID_ARG;
    const size_t vol = (size_t)Z * H * W;
    if (overlap(h, sizeof(float) * (size_t)N * C * vol, Hs, sizeof(float2) * (size_t)N * C * (vol / 2)))
        return HYENA_ERR_INVALID_ARG;
    Fft2dArgs a = {};
    a.v = h;
    a.S = reinterpret_cast<float2*>(Hs);
    a.B = 1;
    a.C = N * C;
    a.W = W / 2;
    a.nq = N * C;
    a.zp = Z;
    a.Hp = H;
    return dispatch_rfft3d(lm, lh, lz, a, (cudaStream_t)stream, false);
}

static hyena_status_t hyena_fftconv3d_gate_forward_circular_impl(bool per_sample, const void* v, const void* const* x, const float* Hs,
                                                     const float* bias, int B, int C, int Z, int H, int W,
                                                     int N, hyena_dtype_t io, void* y, void* workspace,
                                                     size_t ws_bytes, void* stream)
{
    if (!v || !x || !y || !bias || !Hs) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || C < 1 || N < 1 || Z < 1 || H < 1 || W < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_ORDER) return HYENA_ERR_UNSUPPORTED;
    int lz, lh, lm;
    if (!dims3d_circ_ok(Z, H, W, lz, lh, lm)) return HYENA_ERR_UNSUPPORTED;
    if ((long)B * C > (1L << 20) || (long)N * C * Z * H * (per_sample ? B : 1) > (1L << 30))
        return HYENA_ERR_UNSUPPORTED;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !aligned(x[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!aligned(v, 16) || !aligned(y, 16) || !aligned(bias, 4) || !aligned(Hs, 16)) return HYENA_ERR_INVALID_ARG;
    const size_t vol = (size_t)Z * H * W;
    const size_t act = (size_t)B * C * vol * io_bytes(io);
    const size_t spec = sizeof(float2) * (size_t)N * C * (vol / 2) * (per_sample ? (size_t)B : 1);
    const size_t need = hyena_fftconv3d_circular_workspace_size(B, C, Z, H, W);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return HYENA_ERR_WORKSPACE;
    if (overlap(y, act, v, act) || overlap(y, act, bias, sizeof(float) * N * C) || overlap(y, act, Hs, spec) ||
        overlap(y, act, workspace, need) || overlap(workspace, need, v, act) || overlap(workspace, need, Hs, spec))
        return HYENA_ERR_INVALID_ARG;
    for (int n = 0; n < N; ++n)
        if (overlap(y, act, x[n], act) || overlap(workspace, need, x[n], act)) return HYENA_ERR_INVALID_ARG;
    Fft2dArgs a = {};
    a.v = v;
    for (int n = 0; n < kMaxOrder; ++n) a.x[n] = n < N ? x[n] : nullptr;
    a.y = y;
    a.Hs = reinterpret_cast<const float2*>(Hs);
    a.Hs_bstride = per_sample ? (size_t)N * C * (vol / 2) : 0;
    a.bias = bias;
    a.B = B;
    a.C = C;
    a.W = W / 2;
    a.zp = Z;
    a.Hp = H;
    float2* scratch = static_cast<float2*>(workspace);
    cudaStream_t st = (cudaStream_t)stream;
    return io == HYENA_BF16 ? dispatch_fft3d_bf16(lm, lh, lz, a, N, scratch, st, false)
                            : dispatch_fft3d_f32(lm, lh, lz, a, N, scratch, st, false);
}

hyena_status_t hyena_fftconv3d_gate_forward_circular(const void* v, const void* const* x, const float* Hs,
                                                     const float* bias, int B, int C, int Z, int H, int W,
                                                     int N, hyena_dtype_t io, void* y, void* workspace,
                                                     size_t ws_bytes, void* stream)
{
    return hyena_fftconv3d_gate_forward_circular_impl(false, v, x, Hs, bias, B, C, Z, H, W, N, io, y, workspace, ws_bytes, stream);
}

hyena_status_t hyena_fftconv3d_gate_forward_circular_per_sample(const void* v, const void* const* x, const float* Hs,
                                                     const float* bias, int B, int C, int Z, int H, int W,
                                                     int N, hyena_dtype_t io, void* y, void* workspace,
                                                     size_t ws_bytes, void* stream)
{
    return hyena_fftconv3d_gate_forward_circular_impl(true, v, x, Hs, bias, B, C, Z, H, W, N, io, y, workspace, ws_bytes, stream);
}


}  // extern "C"

// ------------------------------------------------------- 2-D backward

namespace {

struct Bwd2dLayout {
    size_t acc, zsave, csave, scratch, total;
    long wcap;
};

// sets: dh spectra per (n, c): B with per-sample spectra, else 1.
// circular: H x W/2 spectrum slots and scratch rows of W/2 slots
Bwd2dLayout bwd2d_layout(int B, int C, int H, int W, int N, int sets = 1, bool circular = false)
{
    Bwd2dLayout l;
    const int Ws = circular ? W / 2 : W;                      // slots per row
    l.wcap = wave_images((long)B * C, H, Ws);
    const size_t slots = (size_t)(circular ? 1 : 2) * H * Ws; // 2H x W (padded) or H x W/2 spectrum slots
    l.acc = 0;
    l.zsave = l.acc + round_up(sizeof(float2) * (size_t)sets * N * C * slots, 256);
    l.csave = l.zsave + round_up(sizeof(float2) * (size_t)N * l.wcap * slots, 256);
    l.scratch = l.csave + round_up(sizeof(float) * (size_t)N * l.wcap * H * W, 256);
    l.total = l.scratch + round_up(sizeof(float2) * (size_t)l.wcap * H * Ws, 256);
    return l;
}

}  // namespace

extern "C" {

size_t hyena_fftconv2d_backward_workspace_size(int B, int C, int H, int W, int N)
{
    if (B < 1 || C < 1 || N < 1 || N > HYENA_MAX_ORDER) return (size_t)-1;
    const int lh = exact_log2(H), lw = exact_log2(W);
    if (lh < kMinLog2H2d || lh > kMaxLog2H2d || lw < kMinLog2W2d || lw > kMaxLog2W2d) return (size_t)-1;
    return bwd2d_layout(B, C, H, W, N).total;
}

size_t hyena_fftconv2d_backward_per_sample_workspace_size(int B, int C, int H, int W, int N)
{
    if (B < 1 || C < 1 || N < 1 || N > HYENA_MAX_ORDER) return (size_t)-1;
    const int lh = exact_log2(H), lw = exact_log2(W);
    if (lh < kMinLog2H2d || lh > kMaxLog2H2d || lw < kMinLog2W2d || lw > kMaxLog2W2d) return (size_t)-1;
    return bwd2d_layout(B, C, H, W, N, B).total;
}

hyena_status_t hyena_fftconv2d_gate_backward(const void* v, const void* const* x, const float* Hs,
                                             const float* bias, const void* dy, int B, int C, int H, int W,
                                             int N, hyena_dtype_t io, void* dv, void* const* dx, float* dh,
                                             float* dbias, void* workspace, size_t ws_bytes, void* stream)
{
    return backward2d_impl(v, x, Hs, false, false, bias, dy, B, C, H, W, N, io, dv, dx, dh, dbias, workspace,
                           ws_bytes, stream);
}

size_t hyena_fftconv2d_backward_circular_workspace_size(int B, int C, int H, int W, int N)
{
    int lh, lm;
    if (B < 1 || C < 1 || N < 1 || N > HYENA_MAX_ORDER || !dims2d_circ_ok(H, W, lh, lm)) return (size_t)-1;
    return bwd2d_layout(B, C, H, W, N, 1, true).total;
}

size_t hyena_fftconv2d_backward_circular_per_sample_workspace_size(int B, int C, int H, int W, int N)
{
    int lh, lm;
    if (B < 1 || C < 1 || N < 1 || N > HYENA_MAX_ORDER || !dims2d_circ_ok(H, W, lh, lm)) return (size_t)-1;
    return bwd2d_layout(B, C, H, W, N, B, true).total;
}

hyena_status_t hyena_fftconv2d_gate_backward_circular_per_sample(const void* v, const void* const* x,
                                                                 const float* Hs, const float* bias,
                                                                 const void* dy, int B, int C, int H, int W,
                                                                 int N, hyena_dtype_t io, void* dv,
                                                                 void* const* dx, float* dh, float* dbias,
                                                                 void* workspace, size_t ws_bytes, void* stream)
{
    return backward2d_impl(v, x, Hs, true, true, bias, dy, B, C, H, W, N, io, dv, dx, dh, dbias, workspace,
                           ws_bytes, stream);
}

hyena_status_t hyena_fftconv2d_gate_backward_circular(const void* v, const void* const* x, const float* Hs,
                                                      const float* bias, const void* dy, int B, int C, int H,
                                                      int W, int N, hyena_dtype_t io, void* dv, void* const* dx,
                                                      float* dh, float* dbias, void* workspace, size_t ws_bytes,
                                                      void* stream)
{
    return backward2d_impl(v, x, Hs, false, true, bias, dy, B, C, H, W, N, io, dv, dx, dh, dbias, workspace,
                           ws_bytes, stream);
}

hyena_status_t hyena_fftconv2d_gate_backward_per_sample(const void* v, const void* const* x, const float* Hs,
                                                        const float* bias, const void* dy, int B, int C, int H,
                                                        int W, int N, hyena_dtype_t io, void* dv,
                                                        void* const* dx, float* dh, float* dbias,
                                                        void* workspace, size_t ws_bytes, void* stream)
{
    return backward2d_impl(v, x, Hs, true, false, bias, dy, B, C, H, W, N, io, dv, dx, dh, dbias, workspace,
                           ws_bytes, stream);
}

}  // extern "C"

namespace {

// per_sample: a spectrum set per sample; circular: the circular recurrence
// (spectra of H x W/2 slots, hyena_filter_rfft2d_circular)
hyena_status_t backward2d_impl(const void* v, const void* const* x, const float* Hs, bool per_sample,
                               bool circular, const float* bias, const void* dy, int B, int C, int H, int W,
                               int N, hyena_dtype_t io, void* dv, void* const* dx, float* dh, float* dbias,
                               void* workspace, size_t ws_bytes, void* stream)
{
    if (!v || !x || !Hs || !bias || !dy || !dv || !dx || !dh || !dbias) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || C < 1 || N < 1 || H < 1 || W < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_ORDER) return HYENA_ERR_UNSUPPORTED;
    int lh = exact_log2(H), lw = exact_log2(W), lm = 0;
    if (circular) {
        if (!dims2d_circ_ok(H, W, lh, lm)) return HYENA_ERR_UNSUPPORTED;
    } else if (lh < kMinLog2H2d || lh > kMaxLog2H2d || lw < kMinLog2W2d || lw > kMaxLog2W2d) {
        return HYENA_ERR_UNSUPPORTED;
    }
    const int sets = per_sample ? B : 1;                     // spectrum sets and dh sets
    const int Ws = circular ? W / 2 : W;                     // spectrum slots per row
    const int RP = circular ? 1 : 2;                         // spectrum rows per grid row
    if ((long)B * C > (1L << 20) || (long)sets * N * C * H > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !dx[n] || !aligned(x[n], 16) || !aligned(dx[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!aligned(v, 16) || !aligned(dy, 16) || !aligned(dv, 16) || !aligned(Hs, 16) || !aligned(dh, 16) ||
        !aligned(bias, 4) || !aligned(dbias, 4))
        return HYENA_ERR_INVALID_ARG;
    const Bwd2dLayout lay = bwd2d_layout(B, C, H, W, N, sets, circular);
    if (!workspace || ws_bytes < lay.total || !aligned(workspace, 256)) return HYENA_ERR_WORKSPACE;

    // every output against every input, the other outputs and the workspace
    const size_t act = (size_t)B * C * H * W * io_bytes(io);
    struct Range { const void* p; size_t n; };
    Range in[kMaxOrder + 5], out[kMaxOrder + 3];
    int ni = 0, no = 0;
    in[ni++] = {v, act};
    in[ni++] = {dy, act};
    in[ni++] = {Hs, sizeof(float2) * (size_t)sets * N * C * RP * H * Ws};
    in[ni++] = {bias, sizeof(float) * N * C};
    in[ni++] = {workspace, lay.total};
    for (int n = 0; n < N; ++n) in[ni++] = {x[n], act};
    out[no++] = {dv, act};
    out[no++] = {dh, sizeof(float) * (size_t)sets * N * C * H * W};
    out[no++] = {dbias, sizeof(float) * N * C};
    for (int n = 0; n < N; ++n) out[no++] = {dx[n], act};
    for (int o = 0; o < no; ++o) {
        for (int i = 0; i < ni; ++i)
            if (overlap(out[o].p, out[o].n, in[i].p, in[i].n)) return HYENA_ERR_INVALID_ARG;
        for (int p = o + 1; p < no; ++p)
            if (overlap(out[o].p, out[o].n, out[p].p, out[p].n)) return HYENA_ERR_INVALID_ARG;
    }

    char* ws = static_cast<char*>(workspace);
    Bwd2dArgs a = {};
    a.f.Hs_bstride = per_sample ? (size_t)N * C * RP * H * Ws : 0;
    a.f.v = v;
    for (int n = 0; n < kMaxOrder; ++n) {
        a.f.x[n] = n < N ? x[n] : nullptr;
        a.dx[n] = n < N ? dx[n] : nullptr;
    }
    a.f.Hs = reinterpret_cast<const float2*>(Hs);
    a.f.bias = bias;
    a.f.S = reinterpret_cast<float2*>(ws + lay.scratch);
    a.f.B = B;
    a.f.C = C;
    a.f.H = H;
    a.f.W = Ws;
    a.dy = dy;
    a.dv = dv;
    a.acc = reinterpret_cast<float2*>(ws + lay.acc);
    a.zsave = reinterpret_cast<float2*>(ws + lay.zsave);
    a.csave = reinterpret_cast<float*>(ws + lay.csave);
    a.dh = dh;
    a.dbias = dbias;
    a.wcap = (int)lay.wcap;
    cudaStream_t st = (cudaStream_t)stream;
    if (circular)
        return io == HYENA_BF16 ? dispatch_bwd2d_circ_bf16(lm, lh, a, N, st)
                                : dispatch_bwd2d_circ_f32(lm, lh, a, N, st);
    return io == HYENA_BF16 ? dispatch_bwd2d_bf16(lw, lh, a, N, st) : dispatch_bwd2d_f32(lw, lh, a, N, st);
}

}  // namespace

// ------------------------------------------------------- 3-D backward

namespace {

// sets: dh spectra per (n, c) (B with per-sample spectra, else 1);
// circular: Z x H x W/2 spectrum slots a volume, else 2Z x 2H x W
Bwd2dLayout bwd3d_layout(int B, int C, int Z, int H, int W, int N, int sets, bool circular)
{
    Bwd2dLayout l;
    const int Ws = circular ? W / 2 : W;
    const int RP = circular ? 1 : 2;
    l.wcap = wave_images_3d((long)B * C, Z, H, Ws, !circular);
    const size_t slots = (size_t)RP * Z * RP * H * Ws;
    l.acc = 0;
    l.zsave = l.acc + round_up(sizeof(float2) * (size_t)sets * N * C * slots, 256);
    l.csave = l.zsave + round_up(sizeof(float2) * (size_t)N * l.wcap * slots, 256);
    l.scratch = l.csave + round_up(sizeof(float) * (size_t)N * l.wcap * Z * H * W, 256);
    l.total = l.scratch + round_up(sizeof(float2) * (size_t)l.wcap * Z * RP * H * Ws, 256);
    return l;
}

bool dims3d_bwd_ok(bool circular, int Z, int H, int W, int& lz, int& lh, int& lm)
{
    if (circular) return dims3d_circ_ok(Z, H, W, lz, lh, lm);
    return dims3d_ok(Z, H, W, lz, lh, lm);
}

size_t bwd3d_workspace(bool circular, int sets, int B, int C, int Z, int H, int W, int N)
{
    int lz, lh, lm;
    if (B < 1 || C < 1 || N < 1 || N > HYENA_MAX_ORDER || !dims3d_bwd_ok(circular, Z, H, W, lz, lh, lm))
        return (size_t)-1;
    return bwd3d_layout(B, C, Z, H, W, N, sets, circular).total;
}

hyena_status_t backward3d_impl(const void* v, const void* const* x, const float* Hs, bool per_sample,
                               bool circular, const float* bias, const void* dy, int B, int C, int Z, int H,
                               int W, int N, hyena_dtype_t io, void* dv, void* const* dx, float* dh,
                               float* dbias, void* workspace, size_t ws_bytes, void* stream)
{
    if (!v || !x || !Hs || !bias || !dy || !dv || !dx || !dh || !dbias) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || C < 1 || N < 1 || Z < 1 || H < 1 || W < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_ORDER) return HYENA_ERR_UNSUPPORTED;
    int lz, lh, lm;
    if (!dims3d_bwd_ok(circular, Z, H, W, lz, lh, lm)) return HYENA_ERR_UNSUPPORTED;
    const int sets = per_sample ? B : 1;
    const int Ws = circular ? W / 2 : W;                     // spectrum slots per row
    const int RP = circular ? 1 : 2;                         // spectrum planes (rows) per grid plane (row)
    if ((long)B * C > (1L << 20) || (long)sets * N * C * Z * H > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !dx[n] || !aligned(x[n], 16) || !aligned(dx[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!aligned(v, 16) || !aligned(dy, 16) || !aligned(dv, 16) || !aligned(Hs, 16) || !aligned(dh, 16) ||
        !aligned(bias, 4) || !aligned(dbias, 4))
        return HYENA_ERR_INVALID_ARG;
    const Bwd2dLayout lay = bwd3d_layout(B, C, Z, H, W, N, sets, circular);
    if (!workspace || ws_bytes < lay.total || !aligned(workspace, 256)) return HYENA_ERR_WORKSPACE;

    // every output against every input, the other outputs and the workspace
    const size_t vol = (size_t)Z * H * W;
    const size_t spec_vol = (size_t)RP * Z * RP * H * Ws;    // spectrum slots a volume
    const size_t act = (size_t)B * C * vol * io_bytes(io);
    struct Range { const void* p; size_t n; };
    Range in[kMaxOrder + 5], out[kMaxOrder + 3];
    int ni = 0, no = 0;
    in[ni++] = {v, act};
    in[ni++] = {dy, act};
    in[ni++] = {Hs, sizeof(float2) * (size_t)sets * N * C * spec_vol};
    in[ni++] = {bias, sizeof(float) * N * C};
    in[ni++] = {workspace, lay.total};
    for (int n = 0; n < N; ++n) in[ni++] = {x[n], act};
    out[no++] = {dv, act};
    out[no++] = {dh, sizeof(float) * (size_t)sets * N * C * vol};
    out[no++] = {dbias, sizeof(float) * N * C};
    for (int n = 0; n < N; ++n) out[no++] = {dx[n], act};
    for (int o = 0; o < no; ++o) {
        for (int i = 0; i < ni; ++i)
            if (overlap(out[o].p, out[o].n, in[i].p, in[i].n)) return HYENA_ERR_INVALID_ARG;
        for (int p = o + 1; p < no; ++p)
            if (overlap(out[o].p, out[o].n, out[p].p, out[p].n)) return HYENA_ERR_INVALID_ARG;
    }

    char* ws = static_cast<char*>(workspace);
    Bwd2dArgs a = {};
    a.f.Hs_bstride = per_sample ? (size_t)N * C * spec_vol : 0;
    a.f.v = v;
    for (int n = 0; n < kMaxOrder; ++n) {
        a.f.x[n] = n < N ? x[n] : nullptr;
        a.dx[n] = n < N ? dx[n] : nullptr;
    }
    a.f.Hs = reinterpret_cast<const float2*>(Hs);
    a.f.bias = bias;
    a.f.S = reinterpret_cast<float2*>(ws + lay.scratch);
    a.f.B = B;
    a.f.C = C;
    a.f.H = Z * H;
    a.f.W = Ws;
    a.f.zp = Z;
    a.f.Hp = H;
    a.dy = dy;
    a.dv = dv;
    a.acc = reinterpret_cast<float2*>(ws + lay.acc);
    a.zsave = reinterpret_cast<float2*>(ws + lay.zsave);
    a.csave = reinterpret_cast<float*>(ws + lay.csave);
    a.dh = dh;
    a.dbias = dbias;
    a.wcap = (int)lay.wcap;
    cudaStream_t st = (cudaStream_t)stream;
    return io == HYENA_BF16 ? dispatch_bwd3d_bf16(lm, lh, lz, a, N, st, !circular)
                            : dispatch_bwd3d_f32(lm, lh, lz, a, N, st, !circular);
}

}  // namespace

extern "C" {

size_t hyena_fftconv3d_backward_workspace_size(int B, int C, int Z, int H, int W, int N)
{
    return bwd3d_workspace(false, 1, B, C, Z, H, W, N);
}

size_t hyena_fftconv3d_backward_per_sample_workspace_size(int B, int C, int Z, int H, int W, int N)
{
    return bwd3d_workspace(false, B, B, C, Z, H, W, N);
}

hyena_status_t hyena_fftconv3d_gate_backward(const void* v, const void* const* x, const float* Hs,
                                             const float* bias, const void* dy, int B, int C, int Z, int H,
                                             int W, int N, hyena_dtype_t io, void* dv, void* const* dx,
                                             float* dh, float* dbias, void* workspace, size_t ws_bytes,
                                             void* stream)
{
    return backward3d_impl(v, x, Hs, false, false, bias, dy, B, C, Z, H, W, N, io, dv, dx, dh, dbias, workspace,
                           ws_bytes, stream);
}

hyena_status_t hyena_fftconv3d_gate_backward_per_sample(const void* v, const void* const* x, const float* Hs,
                                                        const float* bias, const void* dy, int B, int C, int Z,
                                                        int H, int W, int N, hyena_dtype_t io, void* dv,
                                                        void* const* dx, float* dh, float* dbias,
                                                        void* workspace, size_t ws_bytes, void* stream)
{
    return backward3d_impl(v, x, Hs, true, false, bias, dy, B, C, Z, H, W, N, io, dv, dx, dh, dbias, workspace,
                           ws_bytes, stream);
}

size_t hyena_fftconv3d_backward_circular_workspace_size(int B, int C, int Z, int H, int W, int N)
{
    return bwd3d_workspace(true, 1, B, C, Z, H, W, N);
}

size_t hyena_fftconv3d_backward_circular_per_sample_workspace_size(int B, int C, int Z, int H, int W, int N)
{
    return bwd3d_workspace(true, B, B, C, Z, H, W, N);
}

hyena_status_t hyena_fftconv3d_gate_backward_circular(const void* v, const void* const* x, const float* Hs,
                                                      const float* bias, const void* dy, int B, int C, int Z,
                                                      int H, int W, int N, hyena_dtype_t io, void* dv,
                                                      void* const* dx, float* dh, float* dbias, void* workspace,
                                                      size_t ws_bytes, void* stream)
{
    return backward3d_impl(v, x, Hs, false, true, bias, dy, B, C, Z, H, W, N, io, dv, dx, dh, dbias, workspace,
                           ws_bytes, stream);
}

hyena_status_t hyena_fftconv3d_gate_backward_circular_per_sample(const void* v, const void* const* x,
                                                                 const float* Hs, const float* bias,
                                                                 const void* dy, int B, int C, int Z, int H,
                                                                 int W, int N, hyena_dtype_t io, void* dv,
                                                                 void* const* dx, float* dh, float* dbias,
                                                                 void* workspace, size_t ws_bytes, void* stream)
{
    return backward3d_impl(v, x, Hs, true, true, bias, dy, B, C, Z, H, W, N, io, dv, dx, dh, dbias, workspace,
                           ws_bytes, stream);
}

}  // extern "C"
