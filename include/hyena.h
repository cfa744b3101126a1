/*
 * hyena.h -- C ABI of the B200 (sm_100a) Hyena long-convolution library.
 *
 * The operator ("Hyena Hierarchy: Towards Larger Convolutional Language
 * Models", abstract: implicitly parametrised long convolutions interleaved
 * with data-controlled gating), read as the order-N recurrence, per batch
 * element b and channel d:
 *
 *     z_0 = v,   z_n = x_n * (h_n (*) z_{n-1} + b_n * z_{n-1}),   y = z_N
 *
 * where (*) is the causal linear convolution over the whole sequence,
 *     (h (*) u)[t] = sum_{s=0..t} h[s] u[t-s],
 * computed through the convolution theorem ("Long Context Language Models
 * and their Biological Applications with Eric Nguyen - #690", 6:27) on a
 * grid zero-padded to twice its size ("Native Multi-Dimensional
 * Subquadratic Operators via Input Dependent Long Convolutions", Handling
 * Boundaries), and b_n is a per-channel bias (skip) term.
 *
 * Conventions for every entry point:
 *  - All array arguments are DEVICE pointers unless stated otherwise; the
 *    caller allocates and owns every buffer and the stream.  The library
 *    never allocates device memory and never synchronises the stream.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  A returned HYENA_OK means the work was
 *    enqueued; kernel faults surface on the stream like any CUDA error.
 *  - Arrays are dense, row-major, C order, the last index fastest.
 *    Complex arrays hold interleaved (re, im) float pairs (complex64).
 *  - Argument errors are detected on the host before anything is enqueued
 *    and return HYENA_ERR_INVALID_ARG (or HYENA_ERR_UNSUPPORTED for valid
 *    but unimplemented shapes); the GPU is not touched.  A failed launch
 *    returns HYENA_ERR_CUDA; hyena_last_cuda_error() then gives the
 *    cudaError_t value (per calling thread).
 *  - The only global state is per-device kernel attributes (the shared
 *    memory opt-in), set on first use.  Calls are otherwise reentrant.
 *  - v, x_n and y (the activations) may be float32 or bf16 (io); filters,
 *    spectra, biases and filter-network weights are always float32.  All
 *    arithmetic is float32; bf16 outputs are rounded to nearest even.
 */
#ifndef HYENA_B200_H
#define HYENA_B200_H

#include <stddef.h>

#if defined(__GNUC__)
#define HYENA_API __attribute__((visibility("default")))
#else
#define HYENA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HYENA_OK = 0,
    HYENA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment, aliasing */
    HYENA_ERR_UNSUPPORTED = 2,  /* valid arguments this build does not implement */
    HYENA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
    HYENA_ERR_CUDA = 4          /* a CUDA call or launch failed */
} hyena_status_t;

typedef enum { HYENA_F32 = 0, HYENA_BF16 = 1 } hyena_dtype_t;

/* Largest order N accepted by the forward calls. */
#define HYENA_MAX_ORDER 16
/* Largest 1-D length L (a power of two) accepted by the 1-D calls. */
#define HYENA_MAX_LEN (1 << 22)

/* The implicit filter network ("Long Context Language Models ... #690",
 * 4:29: an MLP parametrises the filter).  Reading adopted here: positional
 * features
 *   1-D: phi(i) = [t, sin(2 pi k t), cos(2 pi k t) for k = 1..n_bands],
 *        t = i/L, so n_in = 1 + 2 n_bands;
 *   2-D: phi(iy, ix) = [ty, tx, sin/cos(2 pi k ty) for k = 1..n_bands,
 *        sin/cos(2 pi k tx) for k = 1..n_bands], ty = iy/H, tx = ix/W,
 *        so n_in = 2 + 4 n_bands;
 * three bias-free layers a1 = sin(W1 phi), a2 = sin(W2 a1), a3 = sin(W3 a2)
 * of `width` units, a bias-free head o = Wout a3 with N*D outputs, and the
 * window exp(-alpha_d * i / decay_div) (2-D: exp(-alpha_c (iy+ix)/decay_div)).
 * Filter n of channel d is head row n*D + d.
 * All weight arrays are device float32, row-major [out][in]:
 *   W1 [width][n_in], W2 [width][width], W3 [width][width],
 *   Wout [N*D][width], alpha [D].
 * Limits: 1 <= width <= 64, 0 <= n_bands <= 16, decay_div > 0. */
typedef struct {
    const float* W1;
    const float* W2;
    const float* W3;
    const float* Wout;
    const float* alpha;
    int n_bands;
    int width;
    float decay_div;
} hyena_ffn_t;

/* Human-readable name of a status code (static storage, never NULL). */
HYENA_API const char* hyena_status_string(hyena_status_t status);

/* cudaError_t of the last HYENA_ERR_CUDA returned on this thread (0 if
 * none). */
HYENA_API int hyena_last_cuda_error(void);

/* Number of tensor-core waits in this library's kernels that ran out of
 * time on the current device since the library was loaded (0 when none,
 * -1 if the device could not be queried).  Every such wait is bounded
 * (about two seconds); a kernel whose wait times out records it here,
 * frees its tensor memory and returns without writing its outputs.  The
 * query is a device-to-host copy and so waits for the device. */
HYENA_API int hyena_device_fault_count(void);

/* ---------------------------------------------------------------- 1-D */

/* Implicit filters h [N][D][L] float32 from the filter network (see
 * hyena_ffn_t).  Any L >= 1.  ffn is a HOST pointer to the struct; the
 * arrays it names are device pointers. */
HYENA_API hyena_status_t hyena_filter_gen(const hyena_ffn_t* ffn, int N, int D, int L,
                                float* h, void* stream);

/* Input-dependent filters ("Native Multi-Dimensional Subquadratic Operators
 * via Input Dependent Long Convolutions": Input-Dependent Kernels via
 * Registers and FiLM; Kernel Parameterization).  Per sample b the three
 * sine layers of the filter network are modulated feature-wise (FiLM) and
 * each hidden unit has its own frequency:
 *     a_l = sin(omega_l * (gamma_bl * (W_l a_(l-1)) + beta_bl)),  l = 1..3,
 * then the head and a window: the exponential decay of hyena_ffn_t, or,
 * when sigma is given, the Gaussian exp(-t^2 / (2 sigma_d^2)), t = i/L.
 * The control vectors gamma, beta of each sample come from the model (the
 * pages derive them from register tokens); here they are inputs.  All
 * pointers are device pointers, NULL for the default:
 *   omega  [3][width]     per-unit frequencies (default 1)
 *   gamma  [B][3][width]  FiLM scales (default 1)
 *   beta   [B][3][width]  FiLM shifts (default 0)
 *   sigma  [D]            Gaussian window widths (default: exponential) */
typedef struct {
    const float* omega;
    const float* gamma;
    const float* beta;
    const float* sigma;
} hyena_film_t;

/* Per-sample filters h [B][N][D][L] float32 (1-D).  With every pointer of
 * film NULL each sample's filters equal hyena_filter_gen's.  Their spectra
 * are hyena_filter_rfft of the B*N rows of D filters (N' = B*N); the
 * forward that uses them is hyena_fftconv_gate_forward_per_sample. */
HYENA_API hyena_status_t hyena_filter_gen_film(const hyena_ffn_t* ffn, const hyena_film_t* film,
                                               int B, int N, int D, int L, float* h, void* stream);

/* Filter spectra H [N][D][L] complex64 in the PACKED real-DFT layout: for
 * each h[n][d] zero-padded to 2L ("Handling Boundaries": pad to double the
 * grid so the product of spectra is a linear, non-circular convolution),
 * its 2L-point DFT X has L+1 distinct bins X[0..L]; X[0] and X[L] are real,
 * so they share slot 0 as (X[0], X[L]) and slot k holds X[k] for
 * 1 <= k < L.  Rows are L * 8 bytes (16-byte aligned rows).
 * h is [N][D][L] float32.  L is a power of two, 16 <= L <= HYENA_MAX_LEN.
 * workspace: device scratch of hyena_filter_rfft_workspace_size(N, D, L)
 * bytes, 256-byte aligned (0 -- NULL allowed -- for L <= 16384).
 * Alignment: h 16 bytes, H 16 bytes.  H must not overlap h or the
 * workspace.  The spectrum depends only on the filters: compute it once
 * and reuse it for every batch and every call. */
HYENA_API size_t hyena_filter_rfft_workspace_size(int N, int D, int L);
HYENA_API hyena_status_t hyena_filter_rfft(const float* h, int N, int D, int L,
                                           float* H, void* workspace, size_t ws_bytes,
                                           void* stream);

/* Bytes of workspace hyena_fftconv_gate_forward needs for these sizes
 * (0 when none).  spectrum_given = 1 when the caller passes the cached
 * spectrum H; 0 when it passes the filters h and the spectrum is computed
 * into the workspace first.  Returns (size_t)-1 for invalid sizes. */
HYENA_API size_t hyena_fftconv_workspace_size(int B, int D, int L, int N,
                                    hyena_dtype_t io, int spectrum_given);

/* The fused order-N forward (the recurrence above) over B*D
 * channel-sequences of length L:
 *   v      [B][D][L] io            input z_0
 *   x      HOST array of N device pointers, each [B][D][L] io (x_1..x_N)
 *   h      [N][D][L] float32 filters, or NULL when H is given
 *   H      [N][D][L] packed complex64 spectra (hyena_filter_rfft), or NULL
 *          when h is given; H wins when both are given
 *   bias   [N][D] float32 (b_n)
 *   y      [B][D][L] io output z_N; must not overlap any input or the
 *          workspace
 *   workspace / ws_bytes: device scratch of at least
 *          hyena_fftconv_workspace_size(...) bytes, 256-byte aligned
 *          (NULL / 0 when that size is 0); it must not overlap any input.
 * L is a power of two, 16 <= L <= HYENA_MAX_LEN; 1 <= N <= HYENA_MAX_ORDER.
 * For L <= 16384 one launch runs all N orders with each sequence on one
 * SM; longer sequences take a four-step FFT through the workspace, 2N + 1
 * launches per wave of sequences (one wave's scratch stays in L2).
 * Alignment: v, x_n, y, h, H 16 bytes; bias 4.
 * Returns HYENA_ERR_WORKSPACE if the workspace is too small. */
HYENA_API hyena_status_t hyena_fftconv_gate_forward(const void* v, const void* const* x,
                                          const float* h, const float* H,
                                          const float* bias, int B, int D,
                                          int L, int N, hyena_dtype_t io,
                                          void* y, void* workspace,
                                          size_t ws_bytes, void* stream);

/* The forward with a filter set per sample (input-dependent filters, see
 * hyena_filter_gen_film): H [B][N][D][L] packed complex64, the spectra of
 * sample b's filters at H + b*N*D*L.  Everything else as
 * hyena_fftconv_gate_forward with the spectrum given (the same workspace
 * size).  Sequence (b, d) multiplies by sample b's spectra of channel d. */
HYENA_API hyena_status_t hyena_fftconv_gate_forward_per_sample(const void* v, const void* const* x,
                                                               const float* H, const float* bias,
                                                               int B, int D, int L, int N,
                                                               hyena_dtype_t io, void* y,
                                                               void* workspace, size_t ws_bytes,
                                                               void* stream);

/* Circular mode ("Native Multi-Dimensional Subquadratic Operators via Input
 * Dependent Long Convolutions", Handling Boundaries: circular convolutions
 * for periodic systems, the alternative to zero padding).  The same
 * recurrence with every convolution circular of length L:
 *     (h (*) u)[t] = sum_{s=0..L-1} h[s] u[(t - s) mod L].
 * L is a power of two, 32 <= L <= HYENA_MAX_LEN; other L return
 * HYENA_ERR_UNSUPPORTED.  L <= 16384 runs one launch with each sequence on
 * one SM and needs no workspace; longer L the four-step transform through
 * the workspace, 2N + 1 launches per wave of sequences.
 * hyena_filter_rfft_circular: H [N][D][L/2] complex64, the L-point DFT X of
 * each filter without padding, packed like hyena_filter_rfft's spectra:
 * slot 0 = (X[0], X[L/2]) (both real), slot k = X[k] for 1 <= k < L/2;
 * workspace of hyena_filter_rfft_circular_workspace_size(N, D, L) bytes.
 * hyena_fftconv_gate_forward_circular: v, x_n, y [B][D][L] io, H as above,
 * bias [N][D]; workspace of hyena_fftconv_circular_workspace_size(B, D, L,
 * N) bytes.  Workspaces are 256-byte aligned, NULL / 0 when the size is 0,
 * and must not overlap any argument.  Alignment: h, H, v, x_n, y 16 bytes;
 * bias 4.  The size functions return (size_t)-1 for invalid sizes. */
HYENA_API size_t hyena_filter_rfft_circular_workspace_size(int N, int D, int L);
HYENA_API hyena_status_t hyena_filter_rfft_circular(const float* h, int N, int D, int L, float* H,
                                                    void* workspace, size_t ws_bytes, void* stream);
HYENA_API size_t hyena_fftconv_circular_workspace_size(int B, int D, int L, int N);
HYENA_API hyena_status_t hyena_fftconv_gate_forward_circular(const void* v, const void* const* x,
                                                             const float* H, const float* bias, int B, int D,
                                                             int L, int N, hyena_dtype_t io, void* y,
                                                             void* workspace, size_t ws_bytes, void* stream);

/* The circular forward with a spectrum set per sample (input-dependent
 * filters in circular mode): H [B][N][D][L/2] from hyena_filter_rfft_circular
 * of the B*N rows of D filters, sequence (b, d) multiplied by sample b's
 * spectra.  Everything else (sizes, workspace) as
 * hyena_fftconv_gate_forward_circular. */
HYENA_API hyena_status_t hyena_fftconv_gate_forward_circular_per_sample(const void* v, const void* const* x,
                                                                        const float* H, const float* bias, int B,
                                                                        int D, int L, int N, hyena_dtype_t io,
                                                                        void* y, void* workspace, size_t ws_bytes,
                                                                        void* stream);

/* The backward pass of the circular recurrence (hyena_fftconv_gate_forward_
 * circular), for training: the exact adjoint with every convolution
 * circular of length L, so both sums wrap around:
 *   dx_n = g * c_n,   e = g * x_n,
 *   dh_n[d][s] = sum_b sum_t e[t] z_{n-1}[(t - s) mod L]   (all L lags),
 *   db_n[d] = dh_n[d][0],
 *   dz_{n-1}[u] = sum_t h_n[(t - u) mod L] e[t] + b_n e[u],   dv = dz_0.
 * Arguments as hyena_fftconv_gate_backward with H [N][D][L/2] from
 * hyena_filter_rfft_circular; dh [N][D][L] and dbias [N][D] summed over the
 * batch; workspace of hyena_fftconv_backward_circular_workspace_size(B,
 * D, L, N) bytes (12 N D L S up to L = 16384, S = min(B, 8) batch slices;
 * above, the four-step backward's), 256-byte aligned.  32 <= L <= HYENA_MAX_LEN, a power of two (the size
 * function returns (size_t)-1 otherwise).  Deterministic: two launches up
 * to L = 16384, the four-step launch sequence above. */
HYENA_API size_t hyena_fftconv_backward_circular_workspace_size(int B, int D, int L, int N);
HYENA_API hyena_status_t hyena_fftconv_gate_backward_circular(const void* v, const void* const* x,
                                                              const float* H, const float* bias,
                                                              const void* dy, int B, int D, int L, int N,
                                                              hyena_dtype_t io, void* dv, void* const* dx,
                                                              float* dh, float* dbias, void* workspace,
                                                              size_t ws_bytes, void* stream);

/* The circular backward with a spectrum set per sample: H [B][N][D][L/2]
 * (sample b's set at H + b*N*D*L/2), dh [B][N][D][L] per sample, dbias
 * [N][D] summed over the batch; workspace of
 * hyena_fftconv_backward_circular_per_sample_workspace_size(B, D, L, N)
 * bytes.  Everything else as hyena_fftconv_gate_backward_circular. */
HYENA_API size_t hyena_fftconv_backward_circular_per_sample_workspace_size(int B, int D, int L, int N);
HYENA_API hyena_status_t hyena_fftconv_gate_backward_circular_per_sample(const void* v, const void* const* x,
                                                                         const float* H, const float* bias,
                                                                         const void* dy, int B, int D, int L,
                                                                         int N, hyena_dtype_t io, void* dv,
                                                                         void* const* dx, float* dh,
                                                                         float* dbias, void* workspace,
                                                                         size_t ws_bytes, void* stream);

/* The order-N forward with z spilled to HBM between orders: one launch per
 * order, each reading z_{n-1} (v for n = 1) and writing z_n (y for n = N)
 * to global memory in float32, instead of chaining all orders on chip as
 * hyena_fftconv_gate_forward does for L <= 16384.  The arithmetic of an
 * order is the same as there (same FFT passes, spectral step and gate), so
 * the results agree to float32 rounding.  It exists to measure what keeping
 * the intermediates on chip saves ("Native Multi-Dimensional Subquadratic
 * Operators via Input Dependent Long Convolutions", Implementation: nSubQ,
 * Fused Kernels / Memory Efficiency).
 * Arguments as hyena_fftconv_gate_forward with the cached spectrum H, plus
 *   workspace / ws_bytes: at least hyena_fftconv_spill_workspace_size(B, D,
 *          L, N) bytes (B D L float32 for z, 0 for N = 1), 256-byte
 *          aligned; nothing in it needs to start at zero; it must not
 *          overlap v, x_n, H, bias or y.
 * L is a power of two, 16 <= L <= 16384 (HYENA_ERR_UNSUPPORTED beyond);
 * 1 <= N <= HYENA_MAX_ORDER.  Returns HYENA_ERR_WORKSPACE if the workspace
 * is missing or too small.  The size function returns (size_t)-1 for
 * invalid or unsupported sizes. */
HYENA_API size_t hyena_fftconv_spill_workspace_size(int B, int D, int L, int N);
HYENA_API hyena_status_t hyena_fftconv_gate_forward_spill(const void* v, const void* const* x,
                                                         const float* H, const float* bias,
                                                         int B, int D, int L, int N,
                                                         hyena_dtype_t io, void* y,
                                                         void* workspace, size_t ws_bytes,
                                                         void* stream);

/* A measurement of one FFT level on the two kinds of arithmetic units, used
 * to choose between them: count independent 32-point complex DFTs (x and y
 * [count][32] complex64, 16-byte aligned, not overlapping), each applied
 * reps times in a row to its previous result with the unitary scale
 * 1/sqrt(32) (so four applications give x back).  method 0: the FP32 pipes
 * (in registers, every value through shared memory between repetitions, as
 * a pass of the shared-memory FFTs exchanges); method 1: the tcgen05 tensor
 * cores (128 vectors as a 128 x 64 real matrix times the 64 x 64 real form
 * of the DFT matrix, TF32 with a hi/lo split for float32 accuracy, the
 * accumulator in tensor memory, read back into shared memory every
 * repetition).  The pages point at matrix-multiply hardware for FFT
 * convolutions ("Long Context Language Models ... #690", 7:06); this entry
 * point measures whether a DFT level on it beats the FFT's own level.
 * 1 <= count <= 2^30, reps >= 1. */
HYENA_API hyena_status_t hyena_dft32_stage(const float* x, float* y, long count, int reps, int method,
                                           void* stream);

/* Size of the scratch array built into the library for
 * hyena_fftconv_gate_forward_noalloc (16 MB on every device that loads the
 * library, held until the process exits). */
#define HYENA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* hyena_fftconv_gate_forward without a workspace, for callers that cannot
 * allocate device memory: hosts that plan all device memory at start-up
 * and hand a kernel only its inputs and outputs, and code where a
 * cudaMalloc would synchronise the device or is not allowed.  The pages
 * have no counterpart; this is an interface choice of this library.
 * Same arguments and results as hyena_fftconv_gate_forward with the cached
 * spectrum H (no h, no workspace).  Sequences longer than 16384 use a
 * scratch array inside the library instead of a workspace:
 *  - its device address is looked up (cudaGetSymbolAddress, the caller's
 *    device current) on every call, so it stays right after
 *    cudaDeviceReset; the first call on a device loads the library's
 *    device code there, so make it before any stream capture;
 *  - one sequence's scratch, 8 L bytes, must fit it: L <= 2^21, else
 *    HYENA_ERR_WORKSPACE;
 *  - all calls on a device share it and it keeps the last call's contents
 *    (nothing in it needs to start at zero); calls that overlap on the GPU
 *    (other streams, other host threads) race on it, so order them.
 * Allocates nothing (no cudaMalloc, no cudaFree). */
HYENA_API hyena_status_t hyena_fftconv_gate_forward_noalloc(const void* v, const void* const* x,
                                                            const float* H, const float* bias,
                                                            int B, int D, int L, int N,
                                                            hyena_dtype_t io, void* y,
                                                            void* stream);

/* The backward pass of the order-N forward, for training: the gradients of
 * a scalar loss whose gradient with respect to y is dy.  The pages give
 * the forward only; the gradient is the exact adjoint (chain rule) of the
 * recurrence above, with g = dL/dz_n running back from dy:
 *   dx_n = g * c_n,   e = g * x_n,   (c_n = h_n (*) z_{n-1} + b_n z_{n-1})
 *   dh_n[d][s] = sum_b sum_t e[t] z_{n-1}[t-s],   db_n[d] = dh_n[d][0],
 *   dz_{n-1}[u] = sum_{t>=u} h_n[t-u] e[t] + b_n e[u],   dv = dz_0.
 * Arguments as hyena_fftconv_gate_forward with the cached spectrum H, plus
 *   dy     [B][D][L] io             gradient of the loss with respect to y
 *   dv     [B][D][L] io             out
 *   dx     HOST array of N device pointers, each [B][D][L] io, out
 *   dh     [N][D][L] float32 out    summed over the batch
 *   dbias  [N][D] float32 out       summed over the batch
 *   workspace / ws_bytes: device scratch of at least
 *          hyena_fftconv_backward_workspace_size(B, D, L, N) bytes (20 N D
 *          L S for L <= 16384, S = min(B, 8) batch slices; above, 8 N D L
 *          plus about N * 100 MB + 64 MB for the waves), 256-byte aligned;
 *          nothing in it needs to start at zero.
 * L is a power of two, 16 <= L <= 2^22; 1 <= N <= HYENA_MAX_ORDER.
 * L <= 16384: two launches: a group of threads owns a channel and a slice
 * of the batch (the slice count chosen so that the groups fill the SMs in
 * the fewest rounds) and walks the slice's sequences (the forward again,
 * then the orders backwards), accumulating the slice's dh spectra; a
 * second launch sums each channel's slice spectra in order and inverts
 * the sums.
 * L > 16384 (the four-step transform): per wave of sequences the forward
 * again, saving each order's spectrum and c_n, then per order in reverse a
 * column launch (dx_n, e = g x_n) and a row launch per channel that
 * accumulates the dh spectrum and forms g's; finally the spectra inverted.
 * Both are deterministic (no atomics).
 * Alignment: v, x_n, dy, dv, dx_n, H, dh 16 bytes; bias, dbias 4.  Outputs
 * must not overlap each other, any input or the workspace. */
HYENA_API size_t hyena_fftconv_backward_workspace_size(int B, int D, int L, int N);
HYENA_API hyena_status_t hyena_fftconv_gate_backward(const void* v, const void* const* x,
                                                     const float* H, const float* bias,
                                                     const void* dy, int B, int D, int L, int N,
                                                     hyena_dtype_t io, void* dv, void* const* dx,
                                                     float* dh, float* dbias, void* workspace,
                                                     size_t ws_bytes, void* stream);

/* The backward pass with a spectrum set per sample (input-dependent
 * filters, see hyena_filter_gen_film and
 * hyena_fftconv_gate_forward_per_sample), for training: the same adjoint
 * with sequence (b, d) using sample b's filters, so
 *   H      [B][N][D][L] packed complex64 (sample b's set at H + b*N*D*L)
 *   dh     [B][N][D][L] float32 out, per sample (no sum over the batch):
 *          dh_n[b][d][s] = sum_t e[t] z_{n-1}[t-s] of sequence (b, d)
 *   dbias  [N][D] float32 out, summed over the batch (the bias is shared)
 *   workspace: hyena_fftconv_backward_per_sample_workspace_size(B, D, L, N)
 *          bytes (8 B N D L + 12 N D L for L <= 16384; above, the
 *          four-step backward's with B times the dh spectra), 256-byte
 *          aligned.
 * Everything else, L up to 2^22 included, as hyena_fftconv_gate_backward.
 * Deterministic: each sequence has its own dh spectrum; L <= 16384 takes
 * two launches (the second inverts the B spectra of each (n, d) and sums
 * their lag-0 values into dbias), longer L the four-step launches plus one
 * that sums dbias. */
HYENA_API size_t hyena_fftconv_backward_per_sample_workspace_size(int B, int D, int L, int N);
HYENA_API hyena_status_t hyena_fftconv_gate_backward_per_sample(const void* v, const void* const* x,
                                                                const float* H, const float* bias,
                                                                const void* dy, int B, int D, int L, int N,
                                                                hyena_dtype_t io, void* dv, void* const* dx,
                                                                float* dh, float* dbias, void* workspace,
                                                                size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- 2-D */

/* Implicit 2-D filters h [N][C][H][W] float32 (features and window as in
 * hyena_ffn_t, 2-D form; D = C).  Any H, W >= 1. */
HYENA_API hyena_status_t hyena_filter_gen_2d(const hyena_ffn_t* ffn, int N, int C,
                                   int H, int W, float* h, void* stream);

/* Input-dependent 2-D filters h [B][N][C][H][W] float32: the FiLM
 * modulation of hyena_filter_gen_film on the 2-D filter network; with
 * film->sigma the window is the Gaussian exp(-(ty^2 + tx^2) /
 * (2 sigma_c^2)), ty = iy/H, tx = ix/W, else the separable decay of
 * hyena_filter_gen_2d.  Their spectra are hyena_filter_rfft2d of the B*N
 * rows of C filters; the forward is hyena_fftconv2d_gate_forward_per_sample. */
HYENA_API hyena_status_t hyena_filter_gen_film_2d(const hyena_ffn_t* ffn, const hyena_film_t* film,
                                                  int B, int N, int C, int H, int W, float* h,
                                                  void* stream);

/* 2-D filter spectra Hs [N][C][2H][W] complex64 in the PACKED real 2-D DFT
 * layout, for filters h [N][C][H][W] (offsets 0..H-1 x 0..W-1) zero-padded
 * to 2H x 2W ("Handling Boundaries"; "Native ND Convolution": the N-D FFT):
 * with X[ky][kx] the 2H x 2W DFT (kx = 0..W distinct bins),
 *   slot [ky][kx] = X[ky][kx]                 for 1 <= kx < W,
 *   slot [ky][0]  = F[ky], the 2H-point DFT over y of the complex column
 *                   c[y] = R_y[0] + i R_y[W],
 * where R_y[k] is the 2W-point DFT of row y (R_y[0], R_y[W] are real), so
 *   X[ky][0] = (F[ky] + conj F[-ky]) / 2,  X[ky][W] = (F[ky] - conj F[-ky]) / (2i).
 * H and W are powers of two in [16, 1024].  Alignment 16 bytes; Hs must
 * not overlap h.  No workspace. */
HYENA_API hyena_status_t hyena_filter_rfft2d(const float* h, int N, int C, int H, int W,
                                             float* Hs, void* stream);

/* Bytes of workspace hyena_fftconv2d_gate_forward needs (the spectra when
 * spectrum_given = 0, plus the scratch of one wave of images);
 * (size_t)-1 for invalid sizes. */
HYENA_API size_t hyena_fftconv2d_workspace_size(int B, int C, int H, int W, int N,
                                                hyena_dtype_t io, int spectrum_given);

/* The order-N 2-D forward, per image (b, c):
 *   z_0 = v,  z_n = x_n * (h_n (*) z_{n-1} + b_n z_{n-1}),  y = z_N
 * with (*) the linear 2-D convolution
 *   (h (*) u)[p][q] = sum_{i <= p, j <= q} h[i][j] u[p-i][q-j]
 * computed on the grid zero-padded to 2H x 2W and cropped to H x W.
 *   v, x_n, y [B][C][H][W] io; h [N][C][H][W] float32 or Hs [N][C][2H][W]
 *   (hyena_filter_rfft2d; wins when both are given); bias [N][C];
 *   x is a HOST array of N device pointers.
 * workspace: hyena_fftconv2d_workspace_size(...) bytes, 256-byte aligned.
 * H, W powers of two in [16, 1024]; 1 <= N <= HYENA_MAX_ORDER.
 * Alignment: v, x_n, y, h, Hs 16 bytes; bias 4.  y must not overlap any
 * input or the workspace. */
HYENA_API hyena_status_t hyena_fftconv2d_gate_forward(const void* v, const void* const* x,
                                                      const float* h, const float* Hs,
                                                      const float* bias, int B, int C, int H,
                                                      int W, int N, hyena_dtype_t io, void* y,
                                                      void* workspace, size_t ws_bytes,
                                                      void* stream);

/* The 2-D forward with a spectrum set per sample: Hs [B][N][C][2H][W]
 * (hyena_filter_rfft2d of per-sample filters); otherwise as
 * hyena_fftconv2d_gate_forward with the spectrum given. */
HYENA_API hyena_status_t hyena_fftconv2d_gate_forward_per_sample(const void* v, const void* const* x,
                                                                 const float* Hs, const float* bias,
                                                                 int B, int C, int H, int W, int N,
                                                                 hyena_dtype_t io, void* y,
                                                                 void* workspace, size_t ws_bytes,
                                                                 void* stream);

/* ---------------------------------------------------------------- 3-D */

/* Implicit 3-D filters h [N][C][Z][H][W] float32: the filter network of
 * hyena_ffn_t on per-axis features of the volume,
 *   phi(iz, iy, ix) = [tz, ty, tx, (sin, cos)(2 pi k tz) for k = 1..n_bands,
 *                      the same for ty, then for tx],  t = i / n per axis
 * (W1 is [width][3 + 6 n_bands]), times the separable decay window
 * exp(-alpha_c (iz + iy + ix) / decay_div).  n_bands <= 10 (else
 * HYENA_ERR_UNSUPPORTED).  Any Z, H, W >= 1. */
HYENA_API hyena_status_t hyena_filter_gen_3d(const hyena_ffn_t* ffn, int N, int C, int Z, int H, int W,
                                             float* h, void* stream);

/* Input-dependent 3-D filters h [B][N][C][Z][H][W] float32 ("Native
 * Multi-Dimensional Subquadratic Operators via Input Dependent Long
 * Convolutions": Input-Dependent Kernels via Registers and FiLM, Kernel
 * Parameterization, read on 3-D volumes): per sample b the sine layers of
 * hyena_filter_gen_3d's network are FiLM-modulated as in
 * hyena_filter_gen_film (film: omega [3][width], gamma and beta
 * [B][3][width], device pointers, NULL for 1 / 1 / 0).  Window: with
 * film->sigma [C] the Gaussian exp(-(tz^2 + ty^2 + tx^2) / (2 sigma_c^2)),
 * t = i / n per axis, else the separable decay of hyena_filter_gen_3d.
 * n_bands <= 10; B <= 65535.  Their spectra are hyena_filter_rfft3d of the
 * B*N rows of C filters; the forward is
 * hyena_fftconv3d_gate_forward_per_sample. */
HYENA_API hyena_status_t hyena_filter_gen_film_3d(const hyena_ffn_t* ffn, const hyena_film_t* film,
                                                  int B, int N, int C, int Z, int H, int W, float* h,
                                                  void* stream);

/* 3-D filter spectra Hs [N][C][2Z][2H][W] complex64, for filters h
 * [N][C][Z][H][W] float32 (offsets 0..Z-1 x 0..H-1 x 0..W-1) zero-padded
 * to 2Z x 2H x 2W ("Native Multi-Dimensional Subquadratic Operators via
 * Input Dependent Long Convolutions": Native ND Convolution, Handling
 * Boundaries).  The packing extends the 2-D one by the 2Z-point DFT over
 * z of every slot: with X[kz][ky][kx] the 3-D DFT,
 *   slot [kz][ky][kx] = X[kz][ky][kx]          for 1 <= kx < W,
 *   slot [kz][ky][0]  = A = X0 + i XW,  X0 = X[.][.][0], XW = X[.][.][W],
 * so X0 = (A + conj A') / 2 and XW = (A - conj A') / (2i) with A' the slot
 * at (-kz, -ky).  Z, H, W powers of two in [16, 256]; N*C*Z*H <= 2^30.
 * Alignment 16 bytes; Hs must not overlap h.  No workspace. */
HYENA_API hyena_status_t hyena_filter_rfft3d(const float* h, int N, int C, int Z, int H, int W,
                                             float* Hs, void* stream);

/* Bytes of workspace hyena_fftconv3d_gate_forward needs (the spectra when
 * spectrum_given = 0, plus the scratch of one wave of volumes: Z planes of
 * 2H x W complex slots each); (size_t)-1 for invalid sizes. */
HYENA_API size_t hyena_fftconv3d_workspace_size(int B, int C, int Z, int H, int W, int N,
                                                hyena_dtype_t io, int spectrum_given);

/* The order-N 3-D forward, per volume (b, c):
 *   z_0 = v,  z_n = x_n * (h_n (*) z_{n-1} + b_n z_{n-1}),  y = z_N
 * with (*) the linear 3-D convolution
 *   (h (*) u)[p][q][r] = sum_{i <= p, j <= q, k <= r} h[i][j][k] u[p-i][q-j][r-k]
 * computed on the volume zero-padded to 2Z x 2H x 2W and cropped.
 *   v, x_n, y [B][C][Z][H][W] io; h [N][C][Z][H][W] float32 or Hs
 *   [N][C][2Z][2H][W] (hyena_filter_rfft3d; wins when both are given);
 *   bias [N][C]; x is a HOST array of N device pointers.
 * workspace: hyena_fftconv3d_workspace_size(...) bytes, 256-byte aligned.
 * Z, H, W powers of two in [16, 256]; 1 <= N <= HYENA_MAX_ORDER.
 * Alignment: v, x_n, y, h, Hs 16 bytes; bias 4.  y must not overlap any
 * input or the workspace.  Per volume and order: forward rows, forward
 * columns, the z transform with the spectral multiply and its inverse,
 * inverse columns, inverse rows with the gate (fused with the next
 * order's forward rows). */
HYENA_API hyena_status_t hyena_fftconv3d_gate_forward(const void* v, const void* const* x,
                                                      const float* h, const float* Hs,
                                                      const float* bias, int B, int C, int Z,
                                                      int H, int W, int N, hyena_dtype_t io,
                                                      void* y, void* workspace, size_t ws_bytes,
                                                      void* stream);

/* The 3-D forward with a spectrum set per sample: Hs [B][N][C][2Z][2H][W]
 * (hyena_filter_rfft3d of per-sample filters, e.g. from
 * hyena_filter_gen_film_3d), volume (b, c) multiplied by sample b's
 * spectra of channel c; otherwise as hyena_fftconv3d_gate_forward with the
 * spectrum given (the same workspace size).  B*N*C*Z*H <= 2^30. */
HYENA_API hyena_status_t hyena_fftconv3d_gate_forward_per_sample(const void* v, const void* const* x,
                                                                 const float* Hs, const float* bias,
                                                                 int B, int C, int Z, int H, int W,
                                                                 int N, hyena_dtype_t io, void* y,
                                                                 void* workspace, size_t ws_bytes,
                                                                 void* stream);

/* ------------------------------------------------------- circular 2-D */

/* Circular 2-D filter spectra Hs [N][C][H][W/2] complex64 for filters h
 * [N][C][H][W] (no padding: "Handling Boundaries", circular convolution
 * for periodic systems).  The packing of hyena_filter_rfft2d at H x W:
 * slot [ky][kx] = X[ky][kx] for 1 <= kx < W/2, slot [ky][0] = the H-point
 * DFT over y of R_y[0] + i R_y[W/2] (R_y the W-point DFT of row y).
 * H a power of two in [16, 1024], W in [32, 1024].  Alignment 16 bytes;
 * Hs must not overlap h.  No workspace. */
HYENA_API hyena_status_t hyena_filter_rfft2d_circular(const float* h, int N, int C, int H, int W,
                                                      float* Hs, void* stream);

/* Bytes of workspace hyena_fftconv2d_gate_forward_circular needs (one wave
 * of images, H x W/2 complex slots each); (size_t)-1 for invalid sizes. */
HYENA_API size_t hyena_fftconv2d_circular_workspace_size(int B, int C, int H, int W);

/* The order-N recurrence with circular 2-D convolutions, per image (b, c):
 *   z_n = x_n * (h_n (*) z_{n-1} + b_n z_{n-1}),
 *   (h (*) u)[p][q] = sum_{i, j} h[i][j] u[(p-i) mod H][(q-j) mod W].
 * v, x_n, y [B][C][H][W] io; Hs from hyena_filter_rfft2d_circular; bias
 * [N][C]; x a HOST array of N device pointers.  Sizes as for the spectra;
 * alignment and aliasing as hyena_fftconv2d_gate_forward. */
HYENA_API hyena_status_t hyena_fftconv2d_gate_forward_circular(const void* v, const void* const* x,
                                                               const float* Hs, const float* bias, int B,
                                                               int C, int H, int W, int N, hyena_dtype_t io,
                                                               void* y, void* workspace, size_t ws_bytes,
                                                               void* stream);

/* The circular 2-D forward with a spectrum set per sample: Hs
 * [B][N][C][H][W/2] (hyena_filter_rfft2d_circular of per-sample filters);
 * otherwise as hyena_fftconv2d_gate_forward_circular. */
HYENA_API hyena_status_t hyena_fftconv2d_gate_forward_circular_per_sample(const void* v, const void* const* x,
                                                                          const float* Hs, const float* bias,
                                                                          int B, int C, int H, int W, int N,
                                                                          hyena_dtype_t io, void* y,
                                                                          void* workspace, size_t ws_bytes,
                                                                          void* stream);

/* ------------------------------------------------------- circular 3-D */

/* Circular 3-D filter spectra Hs [N][C][Z][H][W/2] complex64 for filters
 * h [N][C][Z][H][W] (no padding): the circular 2-D packing of every plane
 * followed by the Z-point DFT over z of every slot; slot [kz][ky][0] holds
 * A = X0 + i XM (bins 0 and W/2), X0 = (A + conj A') / 2 and
 * XM = (A - conj A') / (2i), A' the slot at (-kz, -ky).  Z, H powers of two
 * in [16, 256], W in [32, 256].  Alignment 16 bytes; Hs must not overlap h. */
HYENA_API hyena_status_t hyena_filter_rfft3d_circular(const float* h, int N, int C, int Z, int H, int W,
                                                      float* Hs, void* stream);

/* Bytes of workspace hyena_fftconv3d_gate_forward_circular needs (one wave
 * of volumes, Z x H x W/2 complex slots each); (size_t)-1 for invalid sizes. */
HYENA_API size_t hyena_fftconv3d_circular_workspace_size(int B, int C, int Z, int H, int W);

/* The order-N recurrence with circular 3-D convolutions, per volume (b, c):
 *   (h (*) u)[p][q][r] = sum h[i][j][k] u[(p-i) mod Z][(q-j) mod H][(r-k) mod W].
 * v, x_n, y [B][C][Z][H][W] io; Hs from hyena_filter_rfft3d_circular; bias
 * [N][C]; x a HOST array of N device pointers.  Sizes as for the spectra;
 * alignment and aliasing as hyena_fftconv3d_gate_forward. */
HYENA_API hyena_status_t hyena_fftconv3d_gate_forward_circular(const void* v, const void* const* x,
                                                               const float* Hs, const float* bias, int B,
                                                               int C, int Z, int H, int W, int N,
                                                               hyena_dtype_t io, void* y, void* workspace,
                                                               size_t ws_bytes, void* stream);

/* The circular 3-D forward with a spectrum set per sample: Hs
 * [B][N][C][Z][H][W/2] (hyena_filter_rfft3d_circular of per-sample filters,
 * e.g. from hyena_filter_gen_film_3d); otherwise as
 * hyena_fftconv3d_gate_forward_circular.  B*N*C*Z*H <= 2^30. */
HYENA_API hyena_status_t hyena_fftconv3d_gate_forward_circular_per_sample(const void* v, const void* const* x,
                                                                          const float* Hs, const float* bias,
                                                                          int B, int C, int Z, int H, int W,
                                                                          int N, hyena_dtype_t io, void* y,
                                                                          void* workspace, size_t ws_bytes,
                                                                          void* stream);

/* ------------------------------------------------------- 2-D backward */

/* Bytes of workspace hyena_fftconv2d_gate_backward needs: the accumulated
 * dh spectra [N][C][2H][W] complex64, and per wave of images the saved
 * spectra of z_n (N x 2H x W complex), the saved c_n (N x H x W float32)
 * and the scratch (H x W complex); (size_t)-1 for invalid sizes. */
HYENA_API size_t hyena_fftconv2d_backward_workspace_size(int B, int C, int H, int W, int N);

/* Gradients of a scalar loss through the 2-D recurrence of
 * hyena_fftconv2d_gate_forward, given dy = dL/dy [B][C][H][W] (the chain
 * rule; the pages give no training formulas):
 *   dv [B][C][H][W] io, dx = HOST array of N device pointers [B][C][H][W]
 *   io, dh [N][C][H][W] float32 (dL/dh_n, summed over the batch), dbias
 *   [N][C] float32 (= dh_n[0][0]).
 * Inputs as the forward with the spectra Hs [N][C][2H][W] given.  H, W
 * powers of two in [16, 1024].  Alignment: activations, Hs, dh 16 bytes;
 * bias, dbias 4; workspace 256.  Outputs must not overlap any input, each
 * other or the workspace.  Per wave of images: the forward again, saving
 * Z_n and c_n; then per order in reverse, the rows (dx_n, e = g x_n,
 * forward rows of e) and the columns (dh spectrum += E conj(Z_n); g from
 * (conj(H_n) + b_n) E); finally dh and db from the accumulated spectra.
 * Deterministic (no atomics). */
HYENA_API hyena_status_t hyena_fftconv2d_gate_backward(const void* v, const void* const* x, const float* Hs,
                                                       const float* bias, const void* dy, int B, int C, int H,
                                                       int W, int N, hyena_dtype_t io, void* dv,
                                                       void* const* dx, float* dh, float* dbias,
                                                       void* workspace, size_t ws_bytes, void* stream);

/* The 2-D backward with a spectrum set per sample (input-dependent filters,
 * see hyena_filter_gen_film_2d and hyena_fftconv2d_gate_forward_per_sample):
 * image (b, c) uses sample b's filters, so
 *   Hs     [B][N][C][2H][W] (sample b's set at Hs + b*N*C*2H*W)
 *   dh     [B][N][C][H][W] float32 out, per sample (no sum over the batch)
 *   dbias  [N][C] float32 out, summed over the batch (the bias is shared)
 *   workspace: hyena_fftconv2d_backward_per_sample_workspace_size(...)
 *          bytes (B times the dh spectra of the shared backward),
 *          256-byte aligned.
 * Everything else as hyena_fftconv2d_gate_backward; deterministic, one
 * more launch sums dbias over the samples in order. */
HYENA_API size_t hyena_fftconv2d_backward_per_sample_workspace_size(int B, int C, int H, int W, int N);
HYENA_API hyena_status_t hyena_fftconv2d_gate_backward_per_sample(const void* v, const void* const* x,
                                                                  const float* Hs, const float* bias,
                                                                  const void* dy, int B, int C, int H, int W,
                                                                  int N, hyena_dtype_t io, void* dv,
                                                                  void* const* dx, float* dh, float* dbias,
                                                                  void* workspace, size_t ws_bytes,
                                                                  void* stream);

/* The backward of the circular 2-D recurrence (hyena_fftconv2d_gate_forward_
 * circular), for training: the exact adjoint with every 2-D convolution
 * circular on the H x W grid, so both correlations wrap around:
 *   dh_n[c][a][b] = sum_b' sum_{t,s} e[t][s] z_{n-1}[(t - a) mod H][(s - b) mod W],
 *   db_n[c] = dh_n[c][0][0],
 *   dz_{n-1}[u][w] = sum_{t,s} h_n[(t - u) mod H][(s - w) mod W] e[t][s] + b_n e[u][w].
 * Arguments as hyena_fftconv2d_gate_backward with Hs [N][C][H][W/2] from
 * hyena_filter_rfft2d_circular, dh [N][C][H][W] and dbias [N][C] summed
 * over the batch, and a workspace of
 * hyena_fftconv2d_backward_circular_workspace_size(...) bytes, 256-byte
 * aligned.  H a power of two in [16, 1024], W in [32, 1024]. */
HYENA_API size_t hyena_fftconv2d_backward_circular_workspace_size(int B, int C, int H, int W, int N);
HYENA_API hyena_status_t hyena_fftconv2d_gate_backward_circular(const void* v, const void* const* x,
                                                                const float* Hs, const float* bias,
                                                                const void* dy, int B, int C, int H, int W,
                                                                int N, hyena_dtype_t io, void* dv,
                                                                void* const* dx, float* dh, float* dbias,
                                                                void* workspace, size_t ws_bytes, void* stream);

/* The backward of the circular 2-D recurrence with a spectrum set per
 * sample (input-dependent filters, hyena_fftconv2d_gate_forward_circular_
 * per_sample): per sample the circular adjoint above with that sample's
 * filters, so dh is per sample and only the shared bias's gradient is
 * summed over the batch:
 *   dh_{b,n}[c][a][b'] = sum_{t,s} e_b[t][s] z_{b,n-1}[(t - a) mod H][(s - b') mod W],
 *   db_n[c] = sum_b dh_{b,n}[c][0][0].
 * Arguments as hyena_fftconv2d_gate_backward_circular with Hs
 * [B][N][C][H][W/2] (hyena_filter_rfft2d_circular of each sample's
 * filters), dh [B][N][C][H][W] and a workspace of
 * hyena_fftconv2d_backward_circular_per_sample_workspace_size(...) bytes
 * (B times the dh spectra of the shared backward), 256-byte aligned.
 * Deterministic: one more launch sums dbias over the samples in order. */
HYENA_API size_t hyena_fftconv2d_backward_circular_per_sample_workspace_size(int B, int C, int H, int W, int N);
HYENA_API hyena_status_t hyena_fftconv2d_gate_backward_circular_per_sample(
    const void* v, const void* const* x, const float* Hs, const float* bias, const void* dy, int B, int C,
    int H, int W, int N, hyena_dtype_t io, void* dv, void* const* dx, float* dh, float* dbias,
    void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------- 3-D backward */

/* Bytes of workspace hyena_fftconv3d_gate_backward needs: the accumulated
 * dh spectra [N][C][2Z][2H][W] complex64, and per wave of volumes the
 * saved spectra of z_n (N x 2Z x 2H x W complex), the saved c_n (N x Z x H
 * x W float32) and the scratch (Z x 2H x W complex); (size_t)-1 for
 * invalid sizes. */
HYENA_API size_t hyena_fftconv3d_backward_workspace_size(int B, int C, int Z, int H, int W, int N);

/* Gradients of a scalar loss through the 3-D recurrence of
 * hyena_fftconv3d_gate_forward, given dy = dL/dy [B][C][Z][H][W] (the chain
 * rule; the pages give no training formulas):
 *   dv [B][C][Z][H][W] io, dx = HOST array of N device pointers
 *   [B][C][Z][H][W] io, dh [N][C][Z][H][W] float32 (dL/dh_n, summed over
 *   the batch), dbias [N][C] float32 (= dh_n[0][0][0]).
 * Inputs as the forward with the spectra Hs [N][C][2Z][2H][W] given
 * (hyena_filter_rfft3d).  Z, H, W powers of two in [16, 256].  Alignment:
 * activations, Hs, dh 16 bytes; bias, dbias 4; workspace 256.  Outputs
 * must not overlap any input, each other or the workspace.  Per wave of
 * volumes: the forward again, saving the 3-D spectra Z_n and c_n; then per
 * order in reverse, the rows (dx_n, e = g x_n, forward rows of e), the
 * forward columns, the z step (dh spectrum += E conj(Z_n); g from
 * (conj(H_n) + b_n) E) and the inverse columns; finally dh and db from the
 * accumulated spectra.  Deterministic (no atomics). */
HYENA_API hyena_status_t hyena_fftconv3d_gate_backward(const void* v, const void* const* x, const float* Hs,
                                                       const float* bias, const void* dy, int B, int C, int Z,
                                                       int H, int W, int N, hyena_dtype_t io, void* dv,
                                                       void* const* dx, float* dh, float* dbias,
                                                       void* workspace, size_t ws_bytes, void* stream);

/* The 3-D backward with a spectrum set per sample (input-dependent filters,
 * hyena_fftconv3d_gate_forward_per_sample): volume (b, c) uses sample b's
 * filters, so
 *   Hs     [B][N][C][2Z][2H][W] (sample b's set at Hs + b*N*C*2Z*2H*W)
 *   dh     [B][N][C][Z][H][W] float32 out, per sample
 *   dbias  [N][C] float32 out, summed over the batch (the bias is shared)
 *   workspace: hyena_fftconv3d_backward_per_sample_workspace_size(...)
 *          bytes (B times the dh spectra of the shared backward).
 * Everything else as hyena_fftconv3d_gate_backward; deterministic, one
 * more launch sums dbias over the samples in order. */
HYENA_API size_t hyena_fftconv3d_backward_per_sample_workspace_size(int B, int C, int Z, int H, int W, int N);
HYENA_API hyena_status_t hyena_fftconv3d_gate_backward_per_sample(
    const void* v, const void* const* x, const float* Hs, const float* bias, const void* dy, int B, int C,
    int Z, int H, int W, int N, hyena_dtype_t io, void* dv, void* const* dx, float* dh, float* dbias,
    void* workspace, size_t ws_bytes, void* stream);

/* The backward of the circular 3-D recurrence (hyena_fftconv3d_gate_forward_
 * circular): the exact adjoint with every 3-D convolution circular on the
 * Z x H x W grid, so both correlations wrap around:
 *   dh_n[c][a][p][q] = sum_b sum_{t,s,u} e[t][s][u] z_{n-1}[(t-a) mod Z][(s-p) mod H][(u-q) mod W],
 *   db_n[c] = dh_n[c][0][0][0],
 *   dz_{n-1} = the same correlation of e with h_n, plus b_n e.
 * Arguments as hyena_fftconv3d_gate_backward with Hs [N][C][Z][H][W/2]
 * from hyena_filter_rfft3d_circular, dh [N][C][Z][H][W] and dbias [N][C]
 * summed over the batch, and a workspace of
 * hyena_fftconv3d_backward_circular_workspace_size(...) bytes, 256-byte
 * aligned.  Z, H powers of two in [16, 256], W in [32, 256]. */
HYENA_API size_t hyena_fftconv3d_backward_circular_workspace_size(int B, int C, int Z, int H, int W, int N);
HYENA_API hyena_status_t hyena_fftconv3d_gate_backward_circular(
    const void* v, const void* const* x, const float* Hs, const float* bias, const void* dy, int B, int C,
    int Z, int H, int W, int N, hyena_dtype_t io, void* dv, void* const* dx, float* dh, float* dbias,
    void* workspace, size_t ws_bytes, void* stream);

/* The circular 3-D backward with a spectrum set per sample: Hs
 * [B][N][C][Z][H][W/2], dh [B][N][C][Z][H][W] per sample, dbias [N][C]
 * summed over the batch, workspace
 * hyena_fftconv3d_backward_circular_per_sample_workspace_size(...) bytes;
 * otherwise as hyena_fftconv3d_gate_backward_circular. */
HYENA_API size_t hyena_fftconv3d_backward_circular_per_sample_workspace_size(int B, int C, int Z, int H, int W,
                                                                            int N);
HYENA_API hyena_status_t hyena_fftconv3d_gate_backward_circular_per_sample(
    const void* v, const void* const* x, const float* Hs, const float* bias, const void* dy, int B, int C,
    int Z, int H, int W, int N, hyena_dtype_t io, void* dv, void* const* dx, float* dh, float* dbias,
    void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HYENA_B200_H */
