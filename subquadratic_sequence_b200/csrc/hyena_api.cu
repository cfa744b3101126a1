// hyena_api.cu -- the extern "C" entry points declared in include/hyena.h:
// argument validation on the host, kernel selection and launch.
#include <stdint.h>

#include "filter_gen.cuh"
#include "fused1d.cuh"
#include "hyena.h"

using namespace hyena;

namespace {

thread_local int g_last_cuda_error = 0;

hyena_status_t from_cuda(cudaError_t e)
{
    if (e == cudaSuccess) return HYENA_OK;
    g_last_cuda_error = (int)e;
    return HYENA_ERR_CUDA;
}

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

constexpr int kMinLog2 = 4;    // L >= 16
constexpr int kMaxLog2Fused = 14;  // single-CTA path: L <= 16384

size_t io_bytes(hyena_dtype_t io) { return io == HYENA_BF16 ? 2 : 4; }

// ------------------------------------------------------------ launchers

template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes)
{
    if (bytes <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int LOG2M, typename IO>
hyena_status_t launch_fused(const Fused1dArgs& args, cudaStream_t st)
{
    using F = Fft1d<LOG2M>;
    auto kernel = fused1d_kernel<LOG2M, IO>;
    cudaError_t e = allow_smem(kernel, F::SMEM_BYTES);
    if (e != cudaSuccess) return from_cuda(e);
    const long BD = (long)args.B * args.D;
    const unsigned grid = (unsigned)((BD + F::G - 1) / F::G);
    kernel<<<grid, F::THREADS, F::SMEM_BYTES, st>>>(args);
    return from_cuda(cudaGetLastError());
}

template <int LOG2M>
hyena_status_t launch_rfft(const Rfft1dArgs& args, cudaStream_t st)
{
    using F = Fft1d<LOG2M>;
    auto kernel = rfft1d_kernel<LOG2M>;
    cudaError_t e = allow_smem(kernel, F::SMEM_BYTES_FFT);
    if (e != cudaSuccess) return from_cuda(e);
    const unsigned grid = (unsigned)((args.rows + F::G - 1) / F::G);
    kernel<<<grid, F::THREADS, F::SMEM_BYTES_FFT, st>>>(args);
    return from_cuda(cudaGetLastError());
}

template <typename IO>
hyena_status_t dispatch_fused(int log2m, const Fused1dArgs& a, cudaStream_t st)
{
    switch (log2m) {
    case 4: return launch_fused<4, IO>(a, st);
    case 5: return launch_fused<5, IO>(a, st);
    case 6: return launch_fused<6, IO>(a, st);
    case 7: return launch_fused<7, IO>(a, st);
    case 8: return launch_fused<8, IO>(a, st);
    case 9: return launch_fused<9, IO>(a, st);
    case 10: return launch_fused<10, IO>(a, st);
    case 11: return launch_fused<11, IO>(a, st);
    case 12: return launch_fused<12, IO>(a, st);
    case 13: return launch_fused<13, IO>(a, st);
    case 14: return launch_fused<14, IO>(a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
}

hyena_status_t dispatch_rfft(int log2m, const Rfft1dArgs& a, cudaStream_t st)
{
    switch (log2m) {
    case 4: return launch_rfft<4>(a, st);
    case 5: return launch_rfft<5>(a, st);
    case 6: return launch_rfft<6>(a, st);
    case 7: return launch_rfft<7>(a, st);
    case 8: return launch_rfft<8>(a, st);
    case 9: return launch_rfft<9>(a, st);
    case 10: return launch_rfft<10>(a, st);
    case 11: return launch_rfft<11>(a, st);
    case 12: return launch_rfft<12>(a, st);
    case 13: return launch_rfft<13>(a, st);
    case 14: return launch_rfft<14>(a, st);
    default: return HYENA_ERR_UNSUPPORTED;
    }
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

hyena_status_t launch_filter_gen(const hyena_ffn_t* f, int rows, int D, long npos, int L, int Hh,
                                 int Ww, bool two_d, float* h, cudaStream_t st)
{
    FilterGenArgs a;
    a.W1 = f->W1; a.W2 = f->W2; a.W3 = f->W3; a.Wout = f->Wout; a.alpha = f->alpha;
    a.n_in = two_d ? 2 + 4 * f->n_bands : 1 + 2 * f->n_bands;
    a.width = f->width;
    a.rows = rows;
    a.D = D;
    a.L = L; a.Hh = Hh; a.Ww = Ww;
    a.n_bands = f->n_bands;
    a.inv_div = 1.0f / f->decay_div;
    a.h = h;
    const unsigned grid = (unsigned)((npos + kFgTile - 1) / kFgTile);
    cudaError_t e;
    if (two_d) {
        e = allow_smem(filter_gen_kernel<true>, kFgSmemBytes);
        if (e == cudaSuccess) filter_gen_kernel<true><<<grid, kFgThreads, kFgSmemBytes, st>>>(a);
    } else {
        e = allow_smem(filter_gen_kernel<false>, kFgSmemBytes);
        if (e == cudaSuccess) filter_gen_kernel<false><<<grid, kFgThreads, kFgSmemBytes, st>>>(a);
    }
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(cudaGetLastError());
}

// packed spectrum: L complex slots per filter (bins 0 and L share slot 0)
size_t spectrum_bytes(long N, long D, long L) { return sizeof(float2) * N * D * L; }

size_t round_up(size_t n, size_t a) { return (n + a - 1) / a * a; }

}  // namespace

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
    if ((long)N * D > (1L << 30) || (long)N * D * (long)L > (1L << 40)) return HYENA_ERR_UNSUPPORTED;
    return launch_filter_gen(ffn, N * D, D, L, L, 0, 0, false, h, (cudaStream_t)stream);
}

hyena_status_t hyena_filter_gen_2d(const hyena_ffn_t* ffn, int N, int C, int H, int W, float* h,
                                   void* stream)
{
    hyena_status_t s = check_ffn(ffn);
    if (s != HYENA_OK) return s;
    if (!h || N < 1 || C < 1 || H < 1 || W < 1 || !aligned(h, 4)) return HYENA_ERR_INVALID_ARG;
    if ((long)H * W > (1L << 30) || (long)N * C * (long)H * W > (1L << 40)) return HYENA_ERR_UNSUPPORTED;
    return launch_filter_gen(ffn, N * C, C, (long)H * W, 0, H, W, true, h, (cudaStream_t)stream);
}

hyena_status_t hyena_filter_rfft(const float* h, int N, int D, int L, float* H, void* stream)
{
    if (!h || !H || N < 1 || D < 1) return HYENA_ERR_INVALID_ARG;
    int log2m = 0;
    hyena_status_t s = check_len(L, kMaxLog2Fused, &log2m);
    if (s != HYENA_OK) return s;
    if (!aligned(h, 8) || !aligned(H, 16)) return HYENA_ERR_INVALID_ARG;
    if ((long)N * D > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    if (overlap(h, sizeof(float) * N * D * (size_t)L, H, spectrum_bytes(N, D, L)))
        return HYENA_ERR_INVALID_ARG;
    Rfft1dArgs a;
    a.h = h;
    a.H = reinterpret_cast<float2*>(H);
    a.rows = N * D;
    return dispatch_rfft(log2m, a, (cudaStream_t)stream);
}

size_t hyena_fftconv_workspace_size(int B, int D, int L, int N, hyena_dtype_t io,
                                    int spectrum_given)
{
    int log2m = 0;
    if (B < 1 || D < 1 || N < 1 || N > HYENA_MAX_ORDER || (io != HYENA_F32 && io != HYENA_BF16))
        return (size_t)-1;
    if (check_len(L, kMaxLog2Fused, &log2m) != HYENA_OK) return (size_t)-1;
    return spectrum_given ? 0 : round_up(spectrum_bytes(N, D, L), 256);
}

hyena_status_t hyena_fftconv_gate_forward(const void* v, const void* const* x, const float* h,
                                          const float* H, const float* bias, int B, int D, int L,
                                          int N, hyena_dtype_t io, void* y, void* workspace,
                                          size_t ws_bytes, void* stream)
{
    if (!v || !x || !y || !bias || (!h && !H)) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || D < 1 || N < 1 || L < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_ORDER) return HYENA_ERR_UNSUPPORTED;
    int log2m = 0;
    hyena_status_t s = check_len(L, kMaxLog2Fused, &log2m);
    if (s != HYENA_OK) return s;
    if ((long)B * D > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !aligned(x[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!aligned(v, 16) || !aligned(y, 16) || !aligned(bias, 4)) return HYENA_ERR_INVALID_ARG;
    if ((H && !aligned(H, 16)) || (!H && !aligned(h, 8))) return HYENA_ERR_INVALID_ARG;

    const size_t act = (size_t)B * D * L * io_bytes(io);
    const size_t spec = spectrum_bytes(N, D, L);
    const size_t need = H ? 0 : round_up(spec, 256);
    if (need > 0 && (!workspace || ws_bytes < need || !aligned(workspace, 256)))
        return HYENA_ERR_WORKSPACE;
    // y must not overlap anything it is computed from
    if (overlap(y, act, v, act) || overlap(y, act, bias, sizeof(float) * N * D) ||
        (H && overlap(y, act, H, spec)) ||
        (!H && overlap(y, act, h, sizeof(float) * N * D * (size_t)L)) ||
        (need > 0 && overlap(y, act, workspace, need)))
        return HYENA_ERR_INVALID_ARG;
    for (int n = 0; n < N; ++n)
        if (overlap(y, act, x[n], act)) return HYENA_ERR_INVALID_ARG;
    if (!H && overlap(h, sizeof(float) * N * D * (size_t)L, workspace, need))
        return HYENA_ERR_INVALID_ARG;

    cudaStream_t st = (cudaStream_t)stream;
    const float2* spectrum = reinterpret_cast<const float2*>(H);
    if (!H) {
        Rfft1dArgs ra;
        ra.h = h;
        ra.H = reinterpret_cast<float2*>(workspace);
        ra.rows = N * D;
        s = dispatch_rfft(log2m, ra, st);
        if (s != HYENA_OK) return s;
        spectrum = ra.H;
    }
    Fused1dArgs a;
    a.v = v;
    for (int n = 0; n < kMaxOrder; ++n) a.x[n] = n < N ? x[n] : nullptr;
    a.y = y;
    a.H = spectrum;
    a.bias = bias;
    a.B = B;
    a.D = D;
    a.N = N;
    return io == HYENA_BF16 ? dispatch_fused<__nv_bfloat16>(log2m, a, st)
                            : dispatch_fused<float>(log2m, a, st);
}

}  // extern "C"
