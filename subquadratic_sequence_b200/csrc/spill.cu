// spill.cu -- hyena_fftconv_gate_forward_spill: the order-N forward with z
// written to HBM (float32) between orders, one launch per order.  The fused
// forward keeps z on chip across all N orders ("Native Multi-Dimensional
// Subquadratic Operators via Input Dependent Long Convolutions",
// Implementation: nSubQ, Fused Kernels / Memory Efficiency); this variant
// gives the other side of that comparison with the same FFT, spectral and
// gate arithmetic, so the two outputs differ only by the float32 rounding
// of z, which both keep in float32 anyway.
#include <stdint.h>

#include "k_spill.cuh"

using namespace hyena;

namespace {

bool is_aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb)
{
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + nb && b0 < a0 + na;
}

bool sizes_ok(int B, int D, int L, int N, int* log2m)
{
    if (B < 1 || D < 1 || N < 1 || L < 1 || N > HYENA_MAX_ORDER || (long)B * D > (1L << 30)) return false;
    if ((L & (L - 1)) != 0 || L < (1 << kMinLog2) || L > (1 << kMaxLog2Fused)) return false;
    int m = 0;
    while ((1 << m) < L) ++m;
    *log2m = m;
    return true;
}

}  // namespace

extern "C" size_t hyena_fftconv_spill_workspace_size(int B, int D, int L, int N)
{
    int log2m = 0;
    if (!sizes_ok(B, D, L, N, &log2m)) return (size_t)-1;
    return N > 1 ? sizeof(float) * (size_t)B * D * L : 0;
}

extern "C" hyena_status_t hyena_fftconv_gate_forward_spill(const void* v, const void* const* x, const float* H,
                                                          const float* bias, int B, int D, int L, int N,
                                                          hyena_dtype_t io, void* y, void* workspace,
                                                          size_t ws_bytes, void* stream)
{
    if (!v || !x || !y || !bias || !H) return HYENA_ERR_INVALID_ARG;
    if (B < 1 || D < 1 || N < 1 || L < 1) return HYENA_ERR_INVALID_ARG;
    if (io != HYENA_F32 && io != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    int log2m = 0;
    if (!sizes_ok(B, D, L, N, &log2m)) return HYENA_ERR_UNSUPPORTED;
    for (int n = 0; n < N; ++n)
        if (!x[n] || !is_aligned(x[n], 16)) return HYENA_ERR_INVALID_ARG;
    if (!is_aligned(v, 16) || !is_aligned(y, 16) || !is_aligned(H, 16) || !is_aligned(bias, 4))
        return HYENA_ERR_INVALID_ARG;
    const size_t act = (size_t)B * D * L * (io == HYENA_BF16 ? 2 : 4);
    const size_t spec = sizeof(float2) * (size_t)N * D * L;
    const size_t zbytes = sizeof(float) * (size_t)B * D * L;
    if (N > 1) {
        if (!workspace || ws_bytes < zbytes) return HYENA_ERR_WORKSPACE;
        if (!is_aligned(workspace, 256)) return HYENA_ERR_INVALID_ARG;
    }
    const void* ins[3] = {v, H, bias};
    const size_t in_bytes[3] = {act, spec, sizeof(float) * (size_t)N * D};
    for (int i = 0; i < 3; ++i) {
        if (overlaps(y, act, ins[i], in_bytes[i])) return HYENA_ERR_INVALID_ARG;
        if (N > 1 && overlaps(workspace, zbytes, ins[i], in_bytes[i])) return HYENA_ERR_INVALID_ARG;
    }
    for (int n = 0; n < N; ++n) {
        if (overlaps(y, act, x[n], act)) return HYENA_ERR_INVALID_ARG;
        if (N > 1 && overlaps(workspace, zbytes, x[n], act)) return HYENA_ERR_INVALID_ARG;
    }
    if (N > 1 && overlaps(workspace, zbytes, y, act)) return HYENA_ERR_INVALID_ARG;

    cudaStream_t st = (cudaStream_t)stream;
    const float2* Hc = reinterpret_cast<const float2*>(H);
    if (N == 1) {                       // one order: nothing to spill, the fused kernel as is
        Fused1dArgs a = {};
        a.v = v;
        a.x[0] = x[0];
        a.y = y;
        a.H = Hc;
        a.bias = bias;
        a.B = B;
        a.D = D;
        a.N = 1;
        return io == HYENA_BF16 ? dispatch_fused_bf16(log2m, a, st) : dispatch_fused_f32(log2m, a, st);
    }
    for (int n = 0; n < N; ++n) {
        Fused1dOrderArgs a = {};
        a.zin = n == 0 ? v : workspace;
        a.x = x[n];
        a.zout = n == N - 1 ? y : workspace;
        a.H = Hc + (size_t)n * D * L;
        a.bias = bias + (size_t)n * D;
        a.B = B;
        a.D = D;
        hyena_status_t s;
        if (io == HYENA_F32) s = dispatch_order_f32(log2m, a, st);
        else if (n == 0) s = dispatch_order_bf16_first(log2m, a, st);
        else if (n < N - 1) s = dispatch_order_bf16_mid(log2m, a, st);
        else s = dispatch_order_bf16_last(log2m, a, st);
        if (s != HYENA_OK) return s;
    }
    return HYENA_OK;
}
