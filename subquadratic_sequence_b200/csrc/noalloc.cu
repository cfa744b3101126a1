// noalloc.cu -- hyena_fftconv_gate_forward_noalloc: the order-N forward for
// callers that cannot allocate device memory.
//
// Who needs it: hosts whose device memory is planned once at start-up and
// never grown afterwards (inference servers and plugin hosts that hand a
// kernel its inputs and outputs but no workspace), and code that must not
// call cudaMalloc because doing so would synchronise the device or is
// forbidden in that context.  hyena_fftconv_gate_forward needs a workspace
// for sequences longer than 16384 (the four-step FFT scratch); this entry
// point instead uses a scratch array that lives in the library itself.
//
// The scratch is a file-scope __device__ array of HYENA_NOALLOC_SCRATCH_BYTES
// (16 MB), so every GPU that loads the library holds those 16 MB until the
// process exits.  In host code the array's name is only a stand-in for the
// device object: its device address is looked up with cudaGetSymbolAddress,
// with the caller's device current, and passed to the kernels.  The lookup
// runs on every call (a host-side table lookup, no device work), so the
// address stays right when a context is torn down and made again
// (cudaDeviceReset), which may load the array at another address.  The
// first call on a device is the one that loads the library's device code
// there; make it before any stream capture.
//
// Sharing rules: every call on a device uses the same array and leaves the
// last call's contents in it.  Nothing in it needs to start at zero -- each
// wave of the four-step FFT writes its scratch before reading it -- but two
// calls that run on the GPU at the same time (different streams, or
// different host threads without ordering) race on it: order such calls on
// one stream or synchronise between them.
#include <stdint.h>

#include "launch.cuh"

using namespace hyena;

// the built-in scratch (one per device that loads the library)
static __device__ __align__(256) float2 g_noalloc_scratch[HYENA_NOALLOC_SCRATCH_BYTES / sizeof(float2)];

namespace {

constexpr size_t kScratchBytes = HYENA_NOALLOC_SCRATCH_BYTES;
constexpr long kScratchSlots = (long)(kScratchBytes / sizeof(float2));

// Device address of the scratch array on the current device, looked up on
// every call: a cached address would go stale after cudaDeviceReset.
hyena_status_t scratch_address(float2** out)
{
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return from_cuda(e);
    *out = static_cast<float2*>(p);
    return HYENA_OK;
}

bool is_aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb)
{
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + nb && b0 < a0 + na;
}

// The four-step forward, wave by wave, each wave as large as the static
// scratch holds (the same kernels as the workspace path).
template <int LM1, int LM2, typename IO>
hyena_status_t run_waves(FourStepArgs a, int N, float2* scratch, cudaStream_t st)
{
    using FS = FourStep<LM1, LM2>;
    const long nseq = (long)a.B * a.D, per = kScratchSlots / FS::M;
    a.S = scratch;
    a.n_last = N - 1;
    for (long q0 = 0; q0 < nseq; q0 += per) {
        const unsigned nq = (unsigned)(nseq - q0 < per ? nseq - q0 : per);
        a.q0 = (int)q0;
        a.n = 0;
        hyena_status_t s = launch(fourstep_col_kernel<LM1, LM2, IO, 0>, nq * FS::COL_CTAS_PER_SEQ,
                                  FS::COL_THREADS, FS::COL_SMEM, st, a);
        for (int n = 0; n < N && s == HYENA_OK; ++n) {
            a.n = n;
            s = launch(fourstep_row_kernel<LM1, LM2, false>, nq * FS::ROW_CTAS_PER_SEQ,
                       FS::ROW_THREADS, FS::ROW_SMEM, st, a);
            if (s != HYENA_OK) break;
            s = n + 1 < N ? launch(fourstep_col_kernel<LM1, LM2, IO, 1>, nq * FS::COL_CTAS_PER_SEQ,
                                   FS::COL_THREADS, FS::COL_SMEM, st, a)
                          : launch(fourstep_col_kernel<LM1, LM2, IO, 2>, nq * FS::COL_CTAS_PER_SEQ,
                                   FS::COL_THREADS, FS::COL_SMEM, st, a);
        }
        if (s != HYENA_OK) return s;
    }
    return HYENA_OK;
}

template <typename IO>
hyena_status_t run_long(int log2m, const FourStepArgs& a, int N, float2* scratch, cudaStream_t st)
{
    switch (log2m) {
    case 15: return run_waves<7, 8, IO>(a, N, scratch, st);
    case 16: return run_waves<8, 8, IO>(a, N, scratch, st);
    case 17: return run_waves<8, 9, IO>(a, N, scratch, st);
    case 18: return run_waves<8, 10, IO>(a, N, scratch, st);
    case 19: return run_waves<9, 10, IO>(a, N, scratch, st);
    case 20: return run_waves<10, 10, IO>(a, N, scratch, st);
    case 21: return run_waves<10, 11, IO>(a, N, scratch, st);
    default: return HYENA_ERR_WORKSPACE;
    }
}

}  // namespace

extern "C" hyena_status_t hyena_fftconv_gate_forward_noalloc(const void* v, const void* const* x,
                                                             const float* H, const float* bias,
                                                             int B, int D, int L, int N,
                                                             hyena_dtype_t io, void* y,
                                                             void* stream)
{
    if (!v || !x || !y || !bias || !H) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || D < 1 || N < 1 || L < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_ORDER || (long)B * D > (1L << 30)) return HYENA_ERR_UNSUPPORTED;
    if ((L & (L - 1)) != 0 || L < (1 << kMinLog2) || L > (1 << kMaxLog2)) return HYENA_ERR_UNSUPPORTED;
    int log2m = 0;
    while ((1 << log2m) < L) ++log2m;
    // one sequence's scratch (8 L bytes) must fit the built-in array
    if ((size_t)L * sizeof(float2) > kScratchBytes) return HYENA_ERR_WORKSPACE;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !is_aligned(x[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!is_aligned(v, 16) || !is_aligned(y, 16) || !is_aligned(H, 16) || !is_aligned(bias, 4))
        return HYENA_ERR_INVALID_ARG;
    const size_t act = (size_t)B * D * L * (io == HYENA_BF16 ? 2 : 4);
    const size_t spec = sizeof(float2) * (size_t)N * D * L;
    if (overlaps(y, act, v, act) || overlaps(y, act, H, spec) ||
        overlaps(y, act, bias, sizeof(float) * (size_t)N * D))
        return HYENA_ERR_INVALID_ARG;
    for (int n = 0; n < N; ++n)
        if (overlaps(y, act, x[n], act)) return HYENA_ERR_INVALID_ARG;

    cudaStream_t st = (cudaStream_t)stream;
    if (log2m <= kMaxLog2Fused) {       // no scratch at these lengths
        Fused1dArgs a = {};
        a.v = v;
        for (int n = 0; n < kMaxOrder; ++n) a.x[n] = n < N ? x[n] : nullptr;
        a.y = y;
        a.H = reinterpret_cast<const float2*>(H);
        a.bias = bias;
        a.B = B;
        a.D = D;
        a.N = N;
        return io == HYENA_BF16 ? dispatch_fused_bf16(log2m, a, st) : dispatch_fused_f32(log2m, a, st);
    }
    float2* scratch = nullptr;
    hyena_status_t s = scratch_address(&scratch);
    if (s != HYENA_OK) return s;
    FourStepArgs a = {};
    a.v = v;
    for (int n = 0; n < kMaxOrder; ++n) a.x[n] = n < N ? x[n] : nullptr;
    a.y = y;
    a.H = reinterpret_cast<const float2*>(H);
    a.bias = bias;
    a.B = B;
    a.D = D;
    return io == HYENA_BF16 ? run_long<__nv_bfloat16>(log2m, a, N, scratch, st)
                            : run_long<float>(log2m, a, N, scratch, st);
}
