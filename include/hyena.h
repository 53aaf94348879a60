/*
 * hyena.h -- C ABI of libhyena_b200.so: the Hyena implicit long-convolution
 * hot path on NVIDIA B200 (sm_100a).
 *
 * Pages cited (title, section):
 *   [HN] "Hyena: 암묵적 장거리 컨볼루션으로 어텐션을 완전 대체한 서브-이차 모델" --
 *        아키텍처 상세: step 1 (v, x_1, …, x_{N-1} = split(W_proj·x)), step 2 (h(t) = FFN(pos_enc(t))·w(t), w(t) = e^{-αt}),
 *        step 3 (y = x_{N-1} ⊙ (h_{N-1} * (x_{N-2} ⊙ (h_{N-2} * (…))))), and the
 *        ImplicitFilter / hyena_operator code sketch.
 *   [ES] "4. Hyena 상세" -- 어떻게 동작하나요? (filter generator: small MLP with
 *        sinusoidal features and an exponential decay window; FFT convolution:
 *        FFT -> pointwise product -> inverse FFT, O(N log N)).
 *   [ND] "Native Multi-Dimensional Subquadratic Operators via Input Dependent
 *        Long Convolutions" -- 방법론: HyenaND (네이티브 ND 합성곱 via the N-D FFT;
 *        레지스터 및 FiLM; 경계 처리: circular, or non-circular by zero-padding
 *        each axis to double).
 *   [SP] "FFT의 반격: Self-Attention의 효율적 대안" -- 토큰 믹서 구성과 생성 지원
 *        (real FFT -> gate on the n/2+1 bins -> inverse FFT).
 *
 * Conventions for every call:
 *   - Pointers named as device pointers must point to device memory (or
 *     memory the device can address) owned by the caller; the library never
 *     takes ownership and never frees.  Host arrays of device pointers
 *     (x[], H[], Dskip[], W[], b[]) are read during the call only.
 *   - Signals are contiguous, channel-major with unit stride along the
 *     sequence (or the last grid axis): (B, D, L) or (B, D, g0, g1, g2).
 *     bf16 means IEEE bfloat16 bits (uint16); all arithmetic is fp32.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and never synchronises the host, except the
 *     first call on each device (see hyena_init).
 *   - Arguments are checked on the host before anything is launched; a
 *     rejected call returns a status other than HY_OK, launches nothing and
 *     leaves a message for hyena_last_error().  Launch failures are returned
 *     as HY_ERR_CUDA.  Outputs must not alias inputs.
 *   - No C++ exception crosses this boundary.
 */
#ifndef HYENA_B200_H
#define HYENA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HYENA_ABI_VERSION 3

typedef enum hy_status {
    HY_OK = 0,
    HY_ERR_INVALID_ARG = 1,   /* a null pointer, a bad size, aliasing, ... */
    HY_ERR_UNSUPPORTED = 2,   /* a valid request outside what is built    */
    HY_ERR_WORKSPACE = 3,     /* workspace missing or too small           */
    HY_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed      */
    HY_ERR_TIMEOUT = 5        /* a bounded device wait gave up (hyena_device_faults) */
} hy_status;

typedef enum hy_dtype { HY_F32 = 0, HY_BF16 = 1 } hy_dtype;

/* Hidden activation: SiLU, identity, or sine sin(ω x) (the SIREN of [ND]
 * 방법론, 커널 매개변수화, with per-unit frequencies ω). */
typedef enum hy_act { HY_ACT_SILU = 0, HY_ACT_IDENTITY = 1, HY_ACT_SINE = 2 } hy_act;
/* Window on the normalised distance n (t/L or |r|/g): exp(-α n) ([HN] step 2,
 * w(t) = e^{-αt}) or the Gaussian exp(-α n²) ([ND] 커널 합성: 학습 가능한
 * 가우시안 윈도우, α = 1/(2σ²)). */
typedef enum hy_window { HY_WIN_EXP = 0, HY_WIN_GAUSS = 1 } hy_window;

/* Interleaved single-precision complex (same bytes as float2 / complex64). */
typedef struct hy_c32 { float re; float im; } hy_c32;

/* Transform length used for a causal (zero-padded) 1-D convolution of
 * length L: n = 2M with M = max(16, next power of two >= L).  Zero-padding to
 * n >= 2L makes the FFT product a linear convolution ([HN] fft_conv, [ND]
 * 경계 처리).  A filter spectrum row therefore has M + 1 bins; for L a power of
 * two >= 16 that is L + 1. */
int64_t hyena_spectrum_bins(int64_t L);

/* ------------------------------------------------------------------------
 * Filter generator  ([HN] step 2 and ImplicitFilter; [ES]; [ND] FiLM)
 *
 *   1-D:  h[s, o, t] = MLP(PE(t))[o] · w_o(t / L)
 *         PE(t) = [t/L (if include_t), cos(2π j t/L) j=1..F, sin(2π j t/L) j=1..F]
 *   3-D:  h[s, o, p] = MLP_s(PE3(r(p)))[o] · w_o(|r(p)| / g)
 *         on the transform grid of edge S (S = 2g, or g when circular); r(p)
 *         is the signed offset of grid index p per axis (i < S/2 -> i, else
 *         i - S); PE3 = per axis (x, y, z): cos(π j r_a/g), sin(π j r_a/g),
 *         j = 1..F.  Non-circular kernels are zero outside |r_a| <= g - 1.
 *   MLP: layer l maps widths[l] -> widths[l+1], y = W_l x + b_l (W_l row-major
 *   out x in); every layer but the last is followed by `act` (for
 *   HY_ACT_SINE: sin(omega[u] y) per hidden unit u, omega holding every
 *   hidden layer's units in order, or 1 when omega is NULL); when
 *   film_gamma is set, the first hidden layer is modulated per filter set s
 *   before the activation: y <- (1 + gamma[s]) ⊙ y + beta[s].
 *   w_o(n) = exp(-alpha[o] n) (window = HY_WIN_EXP) or exp(-alpha[o] n²)
 *   (HY_WIN_GAUSS).
 * ---------------------------------------------------------------------- */
typedef struct hy_filter_desc {
    int ndim;                /* 1 or 3 */
    int L;                   /* ndim = 1: filter length */
    int grid;                /* ndim = 3: unpadded cube edge g (power of two, 4..64) */
    int circular;            /* ndim = 3: 1 = kernel on the g^3 grid */
    int n_freq;              /* F >= 0 */
    int include_t;           /* ndim = 1: prepend t/L to the encoding */
    int n_layers;            /* 1..4 */
    const int *widths;       /* host, n_layers + 1 entries; widths[0] = input width; hidden <= 128 */
    const float *const *W;   /* host array of n_layers device pointers */
    const float *const *b;   /* host array of n_layers device pointers */
    int act;                 /* hy_act for hidden layers */
    const float *film_gamma; /* device (n_sets, widths[1]) or NULL */
    const float *film_beta;  /* device (n_sets, widths[1]) or NULL (with gamma) */
    const float *alpha;      /* device (widths[n_layers]); >= 0 */
    int n_sets;              /* filter sets s (1 unless FiLM-conditioned) */
    const float *omega;      /* device (Σ hidden widths) sine frequencies, or NULL */
    int window;              /* hy_window */
} hy_filter_desc;

/* Writes h (device, fp32): 1-D (n_sets, n_out, L); 3-D (n_sets, n_out, S, S, S).
 * With at least one 128-position tile per SM the layers run on the tensor
 * cores: both of them for one hidden layer with input width <= 63 and hidden
 * width <= 64, else the last one (after at least one hidden layer of width
 * <= 128).  With fewer tiles, two hidden layers of <= 64 units, an input
 * width <= 127 and at least 256 outputs, all three layers do (one CTA per
 * tile and group of 128-output slices); other small cases stay on the FP32
 * pipes.
 * Their inputs and weights are split into fp16 hi + lo (relative error
 * <= 2^-22, fp32 accumulation), which assumes their magnitudes stay below
 * 65504 (the encodings here are bounded and the hidden units O(1)).  The
 * environment variable HYENA_FILTER_ENGINE=simt keeps every layer on the FP32
 * pipes; =tensor_last puts only the last layer on the tensor cores. */
hy_status hyena_filter_gen(const hy_filter_desc *desc, float *h, void *stream);

/* ------------------------------------------------------------------------
 * HyenaND input conditioning  ([ND] 방법론: HyenaND, 레지스터 및 FiLM을 통한
 * 입력 의존적 커널: R register tokens are processed with each sample; the
 * control variable z(x) is the softmax-weighted mean of their activations
 * and modulates the kernel MLP through FiLM)
 *
 *   l[b, r] = query · reg[b, r, :] (query != NULL) + scores[b, r] (scores != NULL)
 *   w[b, :] = softmax_r(l[b, :]);   z[b, :] = Σ_r w[b, r] reg[b, r, :]
 *   gamma[b, o] = b_film[o] + Σ_c W_film[o, c] z[b, c],         o < H
 *   beta[b, o]  = b_film[H + o] + Σ_c W_film[H + o, c] z[b, c],  o < H
 *
 *   reg: device fp32 (B, R, C), the register activations; query: device
 *   fp32 (C) or NULL; scores: device fp32 (B, R) or NULL (both NULL: the
 *   plain mean); W_film: device fp32 (2H, C) row-major; b_film: device fp32
 *   (2H) or NULL; gamma, beta: device fp32 (B, H) outputs -- the film_gamma
 *   / film_beta of hyena_filter_gen with n_sets = B and H = widths[1].
 *   R <= 1024, C <= 8192.  fp32 arithmetic; the softmax subtracts the
 *   maximum logit.
 * ---------------------------------------------------------------------- */
hy_status hyena_register_film(int B, int R, int C, int H, const float *reg, const float *query,
                              const float *scores, const float *W_film, const float *b_film,
                              float *gamma, float *beta, void *stream);

/* ------------------------------------------------------------------------
 * Filter spectrum  ([HN] fft_conv; [ES] FFT convolution; [ND] N-D FFT)
 *
 *   ndim = 1: dims[0] = L.  Each of `rows` filter rows h[r, 0..L) is
 *             zero-padded to n = 2·M (hyena_spectrum_bins) and
 *             H[r, k] = Σ_t h[r, t] e^{-2πi k t / n}, k = 0..M.
 *             (circular = 1: rows of length L = n, a power of two >= 32,
 *             no padding; L/2 + 1 bins.)
 *   ndim = 3: dims = (g0, g1, g2) unpadded grid; rows are kernels on the
 *             transform grid S_a = 2 g_a (or g_a when circular), row-major;
 *             H[r] = rFFT3(h[r]) with shape (S0, S1, S2/2 + 1).
 *   ws: device workspace of hyena_filter_spectrum_workspace() bytes (may be
 *   NULL when that is 0).  For rows longer than the on-chip transform that
 *   size holds two chunk buffers when the rows take more than one chunk: the
 *   chunks then alternate between `stream` and a second stream the library
 *   creates once per device, joined back to `stream` by events (the call
 *   stays ordered on `stream` and can be captured into a graph; calls from
 *   several host threads take turns on the second stream).  Any workspace
 *   of at least one chunk buffer is accepted and runs on `stream` alone.
 * ---------------------------------------------------------------------- */
size_t hyena_filter_spectrum_workspace(int64_t rows, int ndim, const int *dims, int circular);
hy_status hyena_filter_spectrum(int64_t rows, int ndim, const int *dims, int circular,
                                const float *h, hy_c32 *H, void *ws, size_t ws_bytes,
                                void *stream);

/* ------------------------------------------------------------------------
 * One gated long convolution  ([HN] step 3 for one order; skip term D·u)
 *
 *   y[b,d,t] = gate[b,d,t] · ( Σ_{s<=t} h_d[t-s] u[b,d,s] + Dskip[d] · u[b,d,t] )
 *
 *   u, gate, y: (B, D, L) of dtype dt.  gate may be NULL (no gate), Dskip
 *   may be NULL (no skip).  H: (D, hyena_spectrum_bins(L)) spectra of h_d,
 *   shared across the batch.  ws as for hyena_operator with order 2.
 * ---------------------------------------------------------------------- */
hy_status hyena_fftconv(int B, int D, int L, hy_dtype dt, const void *u, const hy_c32 *H,
                        const float *Dskip, const void *gate, void *y, void *ws,
                        size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * The order-N Hyena operator  ([HN] step 3 gating equation and the
 * hyena_operator sketch; D·u skip inside each order)
 *
 *   z_0 = v;  z_k = x_k ⊙ (h_k * z_{k-1} + D_k ⊙ z_{k-1}),  k = 1..order-1;
 *   y = z_{order-1}.   Each h_k * is causal over the whole sequence.
 *
 *   v, x[k], y: (B, D, L) of dtype dt; x is a host array of order-1 device
 *   pointers; H a host array of order-1 device pointers to (D, bins) spectra;
 *   Dskip a host array of order-1 device pointers to (D) fp32 (the array, or
 *   any entry, may be NULL for no skip).  Intermediate z_k stay fp32.
 *   Sequences with hyena_spectrum_bins(L) - 1 <= 16384 run on chip in one
 *   launch with no workspace; longer ones use the multi-pass path, which
 *   takes hyena_operator_workspace() bytes of device workspace: two chunk
 *   buffers of ~104 MB when the rows take more than one chunk, run as two
 *   chunk pipelines on `stream` and a second stream of the library's, as
 *   for hyena_filter_spectrum; one chunk buffer is the minimum accepted.
 * ---------------------------------------------------------------------- */
size_t hyena_operator_workspace(int order, int B, int D, int L, hy_dtype dt);
hy_status hyena_operator(int order, int B, int D, int L, hy_dtype dt, const void *v,
                         const void *const *x, const hy_c32 *const *H,
                         const float *const *Dskip, void *y, void *ws, size_t ws_bytes,
                         void *stream);

/* ------------------------------------------------------------------------
 * Streaming decode step of the spectral gate with a prefix-FFT cache
 * ([SP] 토큰 믹서 구성과 생성 지원: the cache plays the role of a KV-cache so
 * that autoregressive generation does not recompute the FFT every step).
 *
 *   cache: device (B, H, Dh, n/2 + 1) complex, the spectrum of the prefix
 *   seen so far, X_k = Σ_{m < pos} x[m] e^{-2πi k m / n}: all zeros before
 *   the first token, or a prompt's spectrum from hyena_filter_spectrum
 *   (ndim = 1, dims = {n}, circular = 1, each row the prompt padded with
 *   zeros to n).  One call consumes the token at position pos (0 <= pos <
 *   n): x, x2, y are device (B, H, Dh) values at that position (dt), g the
 *   gate as in spectral_gate.
 *     X_k += x e^{-2πi k pos / n}             (cache updated in place)
 *     y = x2 · (1/n) Σ_{k=0}^{n/2} c_k Re(g_k X_k e^{2πi k pos / n}),
 *   c_0 = c_{n/2} = 1, c_k = 2 otherwise: the output of spectral_gate at
 *   pos for the sequence with every later position zero.  x2 may be NULL.
 *   n a power of two in [2, 2^24]; O(n) work per row per step.
 * ---------------------------------------------------------------------- */
hy_status spectral_gate_decode(int B, int H, int Dh, int n, hy_dtype dt, int64_t pos,
                               const void *x, const hy_c32 *g, int64_t g_batch_stride,
                               const void *x2, hy_c32 *cache, void *y, void *stream);

/* ------------------------------------------------------------------------
 * Backward pass of the operator  ([HN] 아키텍처 상세, step 3, differentiated;
 * the pages train the operator but print no gradient formulas -- these are
 * the derivatives of the recurrence above.)
 *
 *   With z_0 = v, c_k = h_k * z_{k-1} + D_k z_{k-1} (causal), z_k = x_k ⊙ c_k,
 *   y = z_K, and dy = dL/dy, from g_K = dy down to k = 1:
 *     dx_k = g_k ⊙ c_k,   e_k = g_k ⊙ x_k,
 *     g_{k-1}[s] = Σ_{t>=s} h_k[t-s] e_k[t] + D_k e_k[s],
 *     dh_k[d, τ] = Σ_b Σ_{t>=τ} e_k[b,d,t] z_{k-1}[b,d,t-τ]   (τ < L),
 *     dD_k[d]   = Σ_b Σ_t e_k[b,d,t] z_{k-1}[b,d,t],
 *   and dv = g_0.
 *   Inputs as hyena_operator (v, x[k], H[k] = spectra of h_k, Dskip may be
 *   NULL) plus dy (dt, (B, D, L)).  Outputs: dv and dx[k] (dt, (B, D, L));
 *   dh[k] (fp32, (D, L)) and dD[k] (fp32, (D)) -- either array or any entry
 *   may be NULL to skip it.  All arithmetic fp32.  Order 2 with L a power
 *   of two in [512, 8192] (and v, x, dy, dv, dx 16-byte aligned, dh 8-byte
 *   aligned) runs one fused kernel: per row both forward transforms, the two
 *   products and inverse transforms on chip, the sums over t >= s taken as
 *   correlations (spectra times conjugate spectra), dh and dD summed per
 *   channel on chip; a channel's rows are shared by at most two CTAs, which
 *   add their partial sums onto the zeroed dh / dD (two fp32 terms onto zero
 *   commute, so the result is deterministic).  Otherwise the convolutions
 *   are the forward path's (the sums over t >= s as causal convolutions of
 *   the time-reversed e_k) with fp32 intermediates in the workspace;
 *   deterministic (no atomics).
 *   ws: device workspace of hyena_operator_backward_workspace() bytes,
 *   256-byte aligned (fp32 intermediates: 2K + 4 signals and the per-row
 *   spectra of e_k; the fused path does not touch it).
 * ---------------------------------------------------------------------- */
size_t hyena_operator_backward_workspace(int order, int B, int D, int L, hy_dtype dt);
hy_status hyena_operator_backward(int order, int B, int D, int L, hy_dtype dt, const void *v,
                                  const void *const *x, const hy_c32 *const *H,
                                  const float *const *Dskip, const void *dy, void *dv,
                                  void *const *dx, float *const *dh, float *const *dD, void *ws,
                                  size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * hyena_operator_noalloc -- the operator above for callers that cannot
 * allocate device memory.  (The pages have no counterpart: this is a
 * deployment variant, not part of the method.)
 *
 * Who needs it: code that runs where cudaMalloc is off limits -- inside a
 * custom allocator or a memory-pool callback, in a plugin whose host
 * framework owns every device allocation, or in a real-time loop that must
 * not enter the driver's allocator.  Such a caller cannot provide the
 * workspace hyena_operator asks for on long sequences.
 *
 * Same arguments and results as hyena_operator, without ws / ws_bytes.
 * Sequences with hyena_spectrum_bins(L) - 1 <= 16384 run on chip as in
 * hyena_operator (no workspace at all).  Longer ones keep their intermediates
 * in one static device array of 32 MiB that the library reserves on every
 * GPU that loads it, until the process exits; one row needs 8 bytes per
 * complex point, so L <= 1,048,576 (longer is rejected with
 * HY_ERR_WORKSPACE or HY_ERR_UNSUPPORTED).  The call allocates nothing and
 * calls no allocating routine.
 *
 * The first call on a device looks up the array's device address (and, like
 * every entry point, uploads the twiddle tables); make that first call before
 * any stream capture.  Every call shares the one array and leaves its
 * contents behind; no part of it needs to start at zero.  Calls whose
 * execution overlaps on the GPU (other streams, other host threads) race on
 * the array: order them on one stream or serialise them.
 * ---------------------------------------------------------------------- */
hy_status hyena_operator_noalloc(int order, int B, int D, int L, hy_dtype dt, const void *v,
                                 const void *const *x, const hy_c32 *const *H,
                                 const float *const *Dskip, void *y, void *stream);

/* ------------------------------------------------------------------------
 * N-D global convolution with gating  ([ND] 네이티브 ND 합성곱, 경계 처리)
 *
 *   y[b,d,p] = gate[b,d,p] · ( Σ_q K_{b,d}[(p - q) mod S] u[b,d,q]
 *                              + Dskip[d] · u[b,d,p] ),  p, q in the grid
 *   ndim = 3, dims = (g0, g1, g2) powers of two (4..128); S = 2g per axis
 *   (circular = 0: linear convolution) or S = g (circular = 1).
 *   u, gate, y: (B, D, g0, g1, g2) fp32; H: spectra (rFFT3 of K) of shape
 *   (S0, S1, S2/2 + 1) per (sample, channel), sample b at H + b·H_batch_stride
 *   (in hy_c32 units; 0 = shared across samples), channel d at
 *   + d·S0·S1·(S2/2+1).  gate / Dskip may be NULL.
 *   ws: hyena_nd_conv_workspace() bytes: slabs run in chunks of ~80 MB of
 *   transform planes, two chunk buffers when there is more than one chunk
 *   (two chunk pipelines on `stream` and the library's second stream, as
 *   for hyena_filter_spectrum); one chunk buffer is the minimum accepted.
 * ---------------------------------------------------------------------- */
size_t hyena_nd_conv_workspace(int ndim, const int *dims, int B, int D, int circular);
hy_status hyena_nd_conv(int ndim, const int *dims, int B, int D, int circular, const float *u,
                        const hy_c32 *H, int64_t H_batch_stride, const float *Dskip,
                        const float *gate, float *y, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Spectral-gating token mixer  ([SP] real FFT -> diagonal gate on n/2+1
 * bins -> inverse FFT; circular)
 *
 *   y[b,h,c,:] = x2[b,h,c,:] ⊙ irFFT_L( g_{b,h} ⊙ rFFT_L(x[b,h,c,:]) )
 *   x, x2, y: (B, H, Dh, L) of dtype dt, L a power of two in [32, 32768];
 *   g: (H, L/2 + 1) complex per sample, sample b at g + b·g_batch_stride
 *   (0 = shared).  At the DC and Nyquist bins only the real part of the
 *   gated product is kept (the inverse of a real transform).  x2 may be NULL.
 * ---------------------------------------------------------------------- */
hy_status spectral_gate(int B, int H, int Dh, int L, hy_dtype dt, const void *x,
                        const hy_c32 *g, int64_t g_batch_stride, const void *x2, void *y,
                        void *stream);

/* ------------------------------------------------------------------------
 * Input projection  ([HN] 아키텍처 상세, step 1: v, x_1, …, x_{N-1} =
 * split(W_proj · x), a learnable linear map)
 *
 *   out_k[b, d, l] = bias[k·D + d] + Σ_c W[k·D + d, c] · x[b, l, c]
 *   for k = 0 .. n_out-1 (n_out = N for an order-N operator: v, x_1, …),
 *   d < D, l < L, c < C.
 *   x: device (B, L, C) token-major activations; W: device (n_out·D, C)
 *   row-major (the PyTorch Linear layout); bias: device fp32 (n_out·D) or
 *   NULL; out: host array of n_out device pointers, each (B, D, L) -- the
 *   channel-major layout hyena_operator reads, no transpose needed.
 *   x, W, out share dt.  bf16: the library's tcgen05 tensor-core GEMM
 *   (bf16 operands, fp32 accumulation in tensor memory); the bias is added
 *   to the fp32 result in the kernel's epilogue and the sum is rounded to
 *   bf16 once.  fp32: fp32 FMA arithmetic (no TF32), the same fused bias.
 *   x, W, out 16-byte aligned and C·sizeof(dt) a multiple of 16;
 *   n_out·D < 2^30, B·L < 2^31.  No workspace is needed
 *   (hyena_projection_workspace() returns 0; ws may be NULL).
 *   A bounded wait of the GEMM that gives up sets HY_FAULT_PROJECTION
 *   (see hyena_device_faults).
 * ---------------------------------------------------------------------- */
size_t hyena_projection_workspace(void);
hy_status hyena_projection(int B, int L, int C, int D, int n_out, hy_dtype dt, const void *x,
                           const void *W, const float *bias, void *const *out, void *ws,
                           size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Host-buffer variants -- the operator, the N-D convolution and the
 * spectral gate above with the signals in HOST memory.  (The pages have no counterpart: this is the I/O
 * runtime around the method.)
 *
 *   v, x[k], y (operator), u, gate, y (N-D) and x, x2, y (gate) are host
 *   pointers with the layouts of the device entry points; H / g and Dskip
 *   stay device pointers.
 *   Use page-locked host memory (cudaHostAlloc / cudaHostRegister): with
 *   pageable memory the copies still work but do not overlap.  Device
 *   pointers for the signals are rejected (HY_ERR_INVALID_ARG).
 *
 *   The rows (N-D: slabs) are cut into chunks of about 16 MB per signal
 *   (whole batches, or runs of channels / heads within one batch; at least
 *   8 rows on the multi-pass path).  Chunk c is copied in on a library-owned copy stream,
 *   computed on `stream` by the same kernels as the device entry point, and
 *   copied out on a second library-owned copy stream, in a ring of 3 device
 *   slots inside ws -- so the copy in of chunk c+1, the compute of chunk c
 *   and the copy out of chunk c-1 overlap.  Results equal the device entry
 *   point's bit for bit.
 *
 *   ws: device workspace of at least *_host_workspace() bytes, 256-byte
 *   aligned, owned by the caller and not to be touched until `stream` has
 *   passed the call.  The call only enqueues work and returns; `stream`
 *   waits for the last copy out, so y is valid once `stream` is
 *   synchronised.  The host buffers must stay valid until then.  The call
 *   creates a few CUDA events (and, on the first call on a device, the two
 *   copy streams); do not call it during stream capture.
 * ---------------------------------------------------------------------- */
size_t hyena_operator_host_workspace(int order, int B, int D, int L, hy_dtype dt);
hy_status hyena_operator_host(int order, int B, int D, int L, hy_dtype dt, const void *v,
                              const void *const *x, const hy_c32 *const *H,
                              const float *const *Dskip, void *y, void *ws, size_t ws_bytes,
                              void *stream);
size_t hyena_nd_conv_host_workspace(int ndim, const int *dims, int B, int D, int circular);
hy_status hyena_nd_conv_host(int ndim, const int *dims, int B, int D, int circular,
                             const float *u, const hy_c32 *H, int64_t H_batch_stride,
                             const float *Dskip, const float *gate, float *y, void *ws,
                             size_t ws_bytes, void *stream);
size_t spectral_gate_host_workspace(int B, int H, int Dh, int L, hy_dtype dt);
hy_status spectral_gate_host(int B, int H, int Dh, int L, hy_dtype dt, const void *x,
                             const hy_c32 *g, int64_t g_batch_stride, const void *x2, void *y,
                             void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Library state and errors
 * ---------------------------------------------------------------------- */
/* Device faults.  No kernel traps or waits without limit.  The streaming
 * convolution (one order over 16-byte aligned power-of-two rows) stages rows
 * with TMA bulk copies that complete on mbarriers; each wait gives up after
 * about one second of %globaltimer, ORs a bit below into a per-device fault
 * word (a static device variable; nothing is allocated) and the CTA returns
 * at its next row boundary, after a bounded wait for its copies in flight.
 * The tensor-core kernels (projection GEMM, tensor-core convolution, filter
 * generator) bound their pipeline waits the same way and wait for their
 * copies and MMAs in flight before they free tensor memory and return; so do
 * the column passes of the multi-pass convolution, which load their tiles
 * with TMA.
 * The outputs of such a launch are then undefined. */
#define HY_FAULT_STREAM_INPUT 0x1u      /* a row's input copy did not land in time */
#define HY_FAULT_STREAM_GATE 0x2u       /* a row's gate copy did not land in time  */
#define HY_FAULT_PROJECTION 0x4u        /* a wait of the tensor-core projection GEMM ran out */
#define HY_FAULT_TC_CONV 0x8u           /* a wait for the tensor-core convolution's MMAs ran out */
#define HY_FAULT_FILTER_MMA 0x10u       /* a wait for the filter generator's MMAs ran out */
#define HY_FAULT_MULTIPASS 0x20u        /* a column tile of the multi-pass convolution did not land in time */
#define HY_FAULT_SELFTEST 0x80000000u   /* hyena_selftest_bounded_wait ran out      */
/* Reads the current device's fault word into *faults after the work queued on
 * `stream` has finished (the call synchronises that stream); clear != 0 then
 * resets it (queued on `stream`).  Returns HY_ERR_TIMEOUT when any bit was
 * set, HY_OK when none, HY_ERR_INVALID_ARG for a null `faults`.
 *
 * The word is one per device, shared by every stream, host thread and call
 * that runs this library's kernels on the device.  The compute entry points
 * return HY_OK once their kernels are launched, so a wait that gives up
 * during those kernels shows up only here.  Synchronising `stream` does not
 * wait for other streams: a bit may belong to another stream's work, and a
 * clear resets the bits of every caller.  Read (and clear) the word only
 * after all streams that ran the library's kernels on this device have been
 * synchronised (cudaDeviceSynchronize), by one owner of that device. */
hy_status hyena_device_faults(uint32_t *faults, int clear, void *stream);
/* Diagnostic for the failure path: launches one CTA whose wait on an
 * mbarrier that can never complete runs out after limit_us microseconds
 * (1..1000000); it records HY_FAULT_SELFTEST and returns, leaving the
 * context usable.  Read the result with hyena_device_faults. */
hy_status hyena_selftest_bounded_wait(uint32_t limit_us, void *stream);
/* Uploads the constant twiddle tables to the current device and creates the
 * stream and events of the chunk pipelines there.  Called implicitly by the
 * first call on each device; that first call blocks the host briefly and
 * must not be made while a stream is being captured.  */
hy_status hyena_init(void);
/* Message for the last non-OK status returned on this host thread. */
const char *hyena_last_error(void);
const char *hyena_status_string(hy_status s);
int hyena_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HYENA_B200_H */
