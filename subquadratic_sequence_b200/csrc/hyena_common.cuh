// hyena_common.cuh -- register-level building blocks shared by the CUDA
// kernels of the Hyena long-convolution path: complex arithmetic on float2,
// compile-time twiddle multiplies, and an unrolled in-register DFT of a
// power-of-two size R <= 32.
//
// The FFT route follows the convolution theorem as stated in "Long Context
// Language Models and their Biological Applications with Eric Nguyen -
// #690" (6:27): transform, multiply elementwise, transform back.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <type_traits>
#include <utility>

namespace hyena {

// Largest order N (number of long convolutions) one forward call accepts.
constexpr int kMaxOrder = 16;

// ------------------------------------------------------------------ utils

template <typename F, int... Is>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, Is...>)
{
    (f(std::integral_constant<int, Is>{}), ...);
}

// Calls f(std::integral_constant<int, i>) for i = 0 .. N-1, fully unrolled.
template <int N, typename F>
__device__ __forceinline__ void static_for(F&& f)
{
    static_for_impl(f, std::make_integer_sequence<int, N>{});
}

__host__ __device__ constexpr int ilog2(int n) { return n <= 1 ? 0 : 1 + ilog2(n / 2); }

__host__ __device__ constexpr int bitrev(int i, int bits)
{
    int r = 0;
    for (int b = 0; b < bits; ++b) r |= ((i >> b) & 1) << (bits - 1 - b);
    return r;
}

// ---------------------------------------------------------------- complex

__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cconj(float2 a) { return make_float2(a.x, -a.y); }
__device__ __forceinline__ float2 cmul(float2 a, float2 b)
{
    return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
// a * conj(b)
__device__ __forceinline__ float2 cmulc(float2 a, float2 b)
{
    return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.y, b.x, -a.x * b.y));
}
__device__ __forceinline__ float2 mul_i(float2 a) { return make_float2(-a.y, a.x); }   // a * i
__device__ __forceinline__ float2 mul_mi(float2 a) { return make_float2(a.y, -a.x); }  // a * (-i)

// ------------------------------------------------------ constant twiddles

// cos(pi k / 32), k = 0..16 (first quadrant of the 64th roots of unity).
__host__ __device__ constexpr float cos64_q1(int k)
{
    constexpr float t[17] = {
        1.0f,
        0.995184726672196886245f,
        0.980785280403230449126f,
        0.956940335732208864936f,
        0.923879532511286756128f,
        0.881921264348355029713f,
        0.831469612302545237079f,
        0.773010453362736960811f,
        0.707106781186547524401f,
        0.634393284163645498215f,
        0.555570233019602224743f,
        0.471396736825997648556f,
        0.382683432365089771728f,
        0.290284677254462367636f,
        0.195090322016128267848f,
        0.0980171403295606019942f,
        0.0f};
    return t[k];
}

// cos(2 pi q / 64) for any integer q.
__host__ __device__ constexpr float cos64(int q)
{
    q = ((q % 64) + 64) % 64;
    return q <= 16 ? cos64_q1(q)
         : q <= 32 ? -cos64_q1(32 - q)
         : q <= 48 ? -cos64_q1(q - 32)
                   : cos64_q1(64 - q);
}
__host__ __device__ constexpr float sin64(int q) { return cos64(q - 16); }

// a * exp(SIGN * 2 pi i Q / 64), specialised for the trivial angles.
template <int Q, int SIGN>
__device__ __forceinline__ float2 mul_w64(float2 a)
{
    constexpr int q = ((Q % 64) + 64) % 64;
    if constexpr (q == 0) {
        return a;
    } else if constexpr (q == 32) {
        return make_float2(-a.x, -a.y);
    } else if constexpr (q == 16) {
        return SIGN > 0 ? mul_i(a) : mul_mi(a);
    } else if constexpr (q == 48) {
        return SIGN > 0 ? mul_mi(a) : mul_i(a);
    } else if constexpr (q % 16 == 8) {
        // |cos| = |sin| = 1/sqrt(2): two adds and two multiplies
        constexpr float c = cos64(q);
        constexpr float s = SIGN * sin64(q);
        constexpr float r = 0.707106781186547524401f;
        constexpr float sc = c > 0 ? 1.0f : -1.0f;
        constexpr float ss = s > 0 ? 1.0f : -1.0f;
        return make_float2(r * (sc * a.x - ss * a.y), r * (ss * a.x + sc * a.y));
    } else {
        constexpr float c = cos64(q);
        constexpr float s = SIGN * sin64(q);
        return make_float2(fmaf(a.x, c, -a.y * s), fmaf(a.x, s, a.y * c));
    }
}

// 0.0f that depends on `dep`: x - x is not folded under IEEE rules (it is
// NaN for x = inf or NaN), so values computed from it cannot be scheduled
// before `dep` exists.  Used to keep data-independent twiddle arithmetic
// next to the data it multiplies instead of hoisted (and held in registers)
// across whole FFT passes.
__device__ __forceinline__ float zero_after(float dep) { return dep - dep; }

// exp(SIGN * i * pi * num / den) with an exactly representable ratio.
template <int SIGN>
__device__ __forceinline__ float2 expi_pi(float ratio)
{
    float s, c;
    sincospif(ratio, &s, &c);
    return make_float2(c, SIGN * s);
}

// ----------------------------------------------------- in-register DFT

// Unnormalised DFT of R complex values held in registers a[0..R-1]:
//   X[k] = sum_j a[j] exp(SIGN 2 pi i j k / R),  natural order in and out.
// Radix-2 decimation in frequency, fully unrolled, constant twiddles.
//  ZERO_HI : a[R/2 .. R-1] are known to be zero (zero-padded input).
//  HALF_OUT: only X[0 .. R/2-1] are needed; the others are left undefined.
template <int R, int SIGN, bool ZERO_HI = false, bool HALF_OUT = false>
__device__ __forceinline__ void dft(float2* a)
{
    static_assert(R >= 1 && R <= 32 && (R & (R - 1)) == 0, "radix");
    if constexpr (R == 1) {
        return;
    } else {
        constexpr int LOGR = ilog2(R);
        static_for<LOGR>([&](auto st) {
            constexpr int stage = decltype(st)::value;
            constexpr int HALF = R >> (stage + 1);   // butterfly span
            constexpr int TW = 64 / (2 * HALF);      // w_{2 HALF} = w64^TW
            static_for<R / (2 * HALF)>([&](auto sb) {
                constexpr int s = decltype(sb)::value * 2 * HALF;
                static_for<HALF>([&](auto kk) {
                    constexpr int k = decltype(kk)::value;
                    if constexpr (ZERO_HI && stage == 0) {
                        a[s + k + HALF] = mul_w64<k * TW, SIGN>(a[s + k]);
                    } else if constexpr (HALF_OUT && HALF == 1) {
                        a[s + k] = cadd(a[s + k], a[s + k + HALF]);
                    } else {
                        const float2 u = a[s + k], v = a[s + k + HALF];
                        a[s + k] = cadd(u, v);
                        a[s + k + HALF] = mul_w64<k * TW, SIGN>(csub(u, v));
                    }
                });
            });
        });
        // the outputs sit in bit-reversed order: rename registers
        float2 t[R];
        static_for<R>([&](auto ii) {
            constexpr int i = decltype(ii)::value;
            if constexpr (!HALF_OUT || i < R / 2) t[i] = a[bitrev(i, LOGR)];
        });
        static_for<R>([&](auto ii) {
            constexpr int i = decltype(ii)::value;
            if constexpr (!HALF_OUT || i < R / 2) a[i] = t[i];
        });
    }
}

// a[r] *= w^r for r = 1..R-1 (w^0 = 1); powers by recurrence.
template <int R>
__device__ __forceinline__ void apply_twiddle_powers(float2* a, float2 w)
{
    if constexpr (R > 1) {
        float2 wr = w;
        static_for<R - 1>([&](auto ii) {
            constexpr int r = decltype(ii)::value + 1;
            a[r] = cmul(a[r], wr);
            if constexpr (r < R - 1) wr = cmul(wr, w);
        });
    }
}

// ------------------------------------------- programmatic dependent launch

// Every kernel of the library is launched with programmatic stream
// serialisation.  At entry it lets the next kernel in the stream begin
// launching (its CTAs are placed as this grid's CTAs drain, once all of them
// have started), then waits until the previous kernel in the stream has
// completed and its memory operations are visible, before touching global
// memory.  This hides the launch gap between dependent kernels.
__device__ __forceinline__ void grid_dependency_begin()
{
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

// ------------------------------------------------ L2 eviction priority
//
// Data that is read or written once (activations, spectra) streams through
// L2 with evict-first priority; scratch that a following launch reads again
// (the four-step wave scratch, the backward's saved spectra) is kept with
// evict-last priority, so the streams do not push it out to HBM.
__device__ __forceinline__ uint64_t l2_evict_first()
{
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_evict_last()
{
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// read-only load / store of a float2 (or a bf16 pair) with an L2 policy
__device__ __forceinline__ float2 ld_hint(const float2* p, uint64_t pol)
{
    float2 v;
    asm volatile("ld.global.nc.L2::cache_hint.v2.f32 {%0, %1}, [%2], %3;"
                 : "=f"(v.x), "=f"(v.y) : "l"(p), "l"(pol));
    return v;
}
__device__ __forceinline__ __nv_bfloat162 ld_hint(const __nv_bfloat162* p, uint64_t pol)
{
    uint32_t u;
    asm volatile("ld.global.nc.L2::cache_hint.b32 %0, [%1], %2;" : "=r"(u) : "l"(p), "l"(pol));
    __nv_bfloat162 v;
    memcpy(&v, &u, 4);
    return v;
}
// coherent load (the location may have been written earlier in this grid)
__device__ __forceinline__ float2 ld_hint_rw(const float2* p, uint64_t pol)
{
    float2 v;
    asm volatile("ld.global.L2::cache_hint.v2.f32 {%0, %1}, [%2], %3;"
                 : "=f"(v.x), "=f"(v.y) : "l"(p), "l"(pol) : "memory");
    return v;
}
__device__ __forceinline__ float4 ld_hint4(const float4* p, uint64_t pol)
{
    float4 v;
    asm volatile("ld.global.nc.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}
__device__ __forceinline__ float4 ld_hint_rw4(const float4* p, uint64_t pol)
{
    float4 v;
    asm volatile("ld.global.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(pol)
                 : "memory");
    return v;
}
__device__ __forceinline__ void st_hint(float2* p, float2 v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(p), "f"(v.x), "f"(v.y), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_hint(__nv_bfloat162* p, __nv_bfloat162 v, uint64_t pol)
{
    uint32_t u;
    memcpy(&u, &v, 4);
    asm volatile("st.global.L2::cache_hint.b32 [%0], %1, %2;" ::"l"(p), "r"(u), "l"(pol) : "memory");
}
// 16-byte asynchronous global -> shared copy with an L2 policy
__device__ __forceinline__ void cp_async16_hint(void* smem_dst, const void* gmem_src, uint64_t pol)
{
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem_src),
                 "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async_row_hint(void* smem_dst, const void* gmem_src, int bytes, int t,
                                                  int nthreads, uint64_t pol)
{
    char* d = static_cast<char*>(smem_dst);
    const char* s = static_cast<const char*>(gmem_src);
    for (int i = t * 16; i < bytes; i += nthreads * 16) cp_async16_hint(d + i, s + i, pol);
}

// ---------------------------------------------------------------- I/O

// Storage types of v, x_n and y.  Two consecutive real samples are moved
// as one element (one float2, or one bf16 pair).
template <typename IO> struct IoPair;
template <> struct IoPair<float> {
    using T = float2;
    static __device__ __forceinline__ float2 load_smem(const T* p) { return *p; }
    static __device__ __forceinline__ float2 load(const T* p) { return __ldg(p); }
    static __device__ __forceinline__ void store(T* p, float2 v) { *p = v; }
    // the same, streamed with evict-first L2 priority
    static __device__ __forceinline__ float2 load_stream(const T* p, uint64_t pol) { return ld_hint(p, pol); }
    static __device__ __forceinline__ void store_stream(T* p, float2 v, uint64_t pol) { st_hint(p, v, pol); }
};
template <> struct IoPair<__nv_bfloat16> {
    using T = __nv_bfloat162;
    static __device__ __forceinline__ float2 load_smem(const T* p) { return __bfloat1622float2(*p); }
    static __device__ __forceinline__ float2 load(const T* p)
    {
        return __bfloat1622float2(__ldg(p));
    }
    static __device__ __forceinline__ void store(T* p, float2 v)
    {
        *p = __floats2bfloat162_rn(v.x, v.y);  // round to nearest even
    }
    static __device__ __forceinline__ float2 load_stream(const T* p, uint64_t pol)
    {
        return __bfloat1622float2(ld_hint(p, pol));
    }
    static __device__ __forceinline__ void store_stream(T* p, float2 v, uint64_t pol)
    {
        st_hint(p, __floats2bfloat162_rn(v.x, v.y), pol);
    }
};

// ------------------------------------------------------- async copies

// 16-byte global -> shared copy that completes asynchronously (no register
// staging); cp_async_wait_all() blocks until this thread's copies landed.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src)
{
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;\n" ::: "memory");
}
// Cooperative copy of `bytes` (a multiple of 16, both ends 16-byte
// aligned) by `nthreads` threads; thread `t` issues every nthreads-th chunk.
__device__ __forceinline__ void cp_async_row(void* smem_dst, const void* gmem_src, int bytes, int t,
                                             int nthreads)
{
    char* d = static_cast<char*>(smem_dst);
    const char* s = static_cast<const char*>(gmem_src);
    for (int i = t * 16; i < bytes; i += nthreads * 16) cp_async16(d + i, s + i);
}

// Shared-memory index with one float2 of padding per 16: strided Stockham
// writes then hit distinct banks.
__device__ __forceinline__ int pad16(int i) { return i + (i >> 4); }
__host__ __device__ constexpr int padded_size(int n) { return n + n / 16; }

// pad16(i + r * S) given pi = pad16(i), for a compile-time stride S: when S
// is a multiple of 16 the padding of the offset is a constant, so the whole
// index is pi plus an immediate.
template <int S>
__device__ __forceinline__ int pad16_at(int i, int pi, int r)
{
    if constexpr (S % 16 == 0) return pi + r * (S + S / 16);
    else return pad16(i + r * S);
}

}  // namespace hyena
