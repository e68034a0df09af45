/*
 * nvfp4_gdn.h -- C ABI of the B200 (sm_100a) NVFP4 W4A4 Gated DeltaNet layer forward.
 *
 * The method is the one described by the web pages on "Why Gated DeltaNet
 * Survives 4-Bit Quantization: NVFP4 W4A4 for the Recurrent Half of a Hybrid
 * 27B LLM" (a review page at jaehun.me and the paper's abstract):
 *   - NVFP4: E2M1 4-bit values, one E4M3 scale per 16-element block and one
 *     FP32 scale per tensor (review page, background section, paper sec.1);
 *   - W4A4 linear layers, the GDN in_proj fused into one GEMM whose modules
 *     share one global weight scale (review page, paper sec.6; abstract);
 *   - gates, Eq.(1): g = -exp(A_log) softplus(a + dt_bias), alpha = e^g,
 *     beta = sigmoid(b) (review page, paper sec.2);
 *   - the delta rule, Eq.(2): S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T,
 *     o_t = S_t^T (q_t / sqrt(K)) (review page, background, paper sec.1).
 *
 * Conventions shared by every call:
 *   - Pointers named in a call are DEVICE pointers owned by the caller unless
 *     the comment says host; the library allocates no device memory.  Scratch
 *     ("workspace") is sized by the matching *_workspace_size() call and
 *     passed in; it must stay valid until the stream reaches the call.  The
 *     one exception is gdn_scan_noalloc, which keeps its scratch in a fixed
 *     array inside the library (see its comment).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and launches only this library's kernels (workspace
 *     words that must start at zero are cleared by one of them, not by a
 *     memset).
 *   - Arguments are validated on the host before anything is launched; a
 *     rejected call launches nothing and returns a non-OK status.  The
 *     message of the last failure on the calling host thread is returned by
 *     nvfp4_last_error().  Nothing throws across this ABI.
 *   - Device-side failures (a bounded wait that ran out) set a device error
 *     word; nvfp4_check_device_error() synchronises the stream and reports
 *     (and clears) it.
 *   - Row-major matrices; `ld` arguments are in elements.
 */
#ifndef NVFP4_GDN_H
#define NVFP4_GDN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,       /* null pointer, negative or zero size, bad enum */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside what the kernels cover */
    NVFP4_ERR_MISALIGNED = 3,        /* pointer or leading dimension not 16-byte aligned */
    NVFP4_ERR_CUDA = 4,              /* a CUDA runtime / driver call failed */
    NVFP4_ERR_TIMEOUT = 5,           /* a kernel's bounded wait ran out (device error word) */
    NVFP4_ERR_WORKSPACE = 6          /* workspace missing or smaller than required */
} nvfp4_status;

typedef void* nvfp4_stream_t; /* cudaStream_t */

enum { NVFP4_DTYPE_BF16 = 0, NVFP4_DTYPE_FP32 = 1 };
enum { NVFP4_QUANT_COMPUTE_SCALE = 0, NVFP4_QUANT_GIVEN_SCALE = 1, NVFP4_QUANT_AMAX_ONLY = 2,
       NVFP4_QUANT_FROM_AMAX = 3 };
enum { GDN_FORM_PAGES = 0, GDN_FORM_STANDARD = 1 };
enum { GDN_SCAN_AUTO = 0, GDN_SCAN_RECURRENT = 1, GDN_SCAN_CHUNKED = 2 };

/* An NVFP4 matrix [rows x cols] (cols % 64 == 0).
 *   codes: rows * cols / 2 bytes, row-major, two E2M1 codes per byte (element
 *          2i in the low nibble), code bits sign|e1 e0|m.  16-byte aligned.
 *   sf:    nvfp4_sf_bytes(rows, cols) bytes of E4M3 block scales in the
 *          tensor-core atom layout: 512-byte atoms covering 128 rows x 4
 *          blocks (64 columns), atoms ordered (row block, column block) with
 *          the column block fastest; the byte of (row r, block j) inside an
 *          atom is at (r % 32) * 16 + ((r / 32) % 4) * 4 + j % 4.  Rows are
 *          padded to a multiple of 128; the quantiser writes 0 in the pad.
 *   global_scale: one float, the per-tensor dequantisation multiplier S, so
 *          that x ~ e2m1(code) * e4m3(sf) * S.                              */
typedef struct {
    uint8_t* codes;
    uint8_t* sf;
    float* global_scale;
    int64_t rows;
    int64_t cols;
} nvfp4_tensor;

/* Head geometry of one GDN layer.  Value head h reads key head h * Hk / Hv. */
typedef struct {
    int32_t Hk; /* key heads */
    int32_t Hv; /* value heads (a multiple of Hk) */
    int32_t K;  /* key head dim: 64 or 128 */
    int32_t V;  /* value head dim: 64 or 128 */
} gdn_dims;

/* ---------------------------------------------------------------- errors -- */
NVFP4_API const char* nvfp4_last_error(void);
/* Synchronises `stream`, then returns NVFP4_ERR_TIMEOUT if any kernel of this
 * library recorded a failed bounded wait on the current device since the last
 * check (and clears the record), else NVFP4_OK (or NVFP4_ERR_CUDA). */
NVFP4_API nvfp4_status nvfp4_check_device_error(nvfp4_stream_t stream);
/* Library version, "major.minor.patch". Host string, static storage. */
NVFP4_API const char* nvfp4_version(void);
/* Test hook for the failure path above (the pages have no counterpart): launches
 * one thread on `stream` that waits on a barrier nothing ever arrives on, with a
 * bounded wait of `budget_cycles` SM clocks (1 .. 2^30), after which it records a
 * failure in the device error word and returns -- the same path every kernel of
 * the library takes when a wait runs out.  The next nvfp4_check_device_error()
 * then reports NVFP4_ERR_TIMEOUT and the CUDA context stays usable.
 * NVFP4_ERR_INVALID_ARG for a budget outside the range. */
NVFP4_API nvfp4_status nvfp4_selftest_wait_timeout(uint32_t budget_cycles, nvfp4_stream_t stream);

/* ------------------------------------------------------------ quantiser -- */
/* Bytes of the scale-factor buffer of an NVFP4 [rows x cols] matrix. */
NVFP4_API size_t nvfp4_sf_bytes(int64_t rows, int64_t cols);
/* Bytes of workspace nvfp4_quantize needs (one amax word, padded). */
NVFP4_API size_t nvfp4_quantize_workspace_size(void);

/* Online NVFP4 quantisation of x [rows x cols] (review page, background /
 * paper sec.1: E2M1 values, E4M3 per-16 scales, FP32 per-tensor scale; the
 * per-tensor scale is computed from the tensor at run time).
 *   x:       device, bf16 or fp32 (x_dtype), row pitch `ld` elements; x and
 *            ld * element size 16-byte aligned; finite values.
 *   out:     host struct describing device buffers (codes, sf, global_scale);
 *            out->rows == rows, out->cols == cols.
 *   flags:   NVFP4_QUANT_COMPUTE_SCALE: S = amax(|x|) / 2688 (S = 1 when
 *            amax < 2^-100) is computed on the device and written to
 *            *out->global_scale;  NVFP4_QUANT_GIVEN_SCALE: the value already
 *            in *out->global_scale is used (harmonised weight scales).
 *            The per-tensor scale of a tensor split across GPUs (rows of a
 *            sequence on several ranks) takes two calls around a collective:
 *            NVFP4_QUANT_AMAX_ONLY sets workspace word 0 to the float bits of
 *            max|x| and writes nothing else; after a max all-reduce of that
 *            word over the ranks (as 32-bit integers: non-negative floats order
 *            as their bits), NVFP4_QUANT_FROM_AMAX quantises with S formed on
 *            the device from word 0 as in COMPUTE_SCALE and writes S to
 *            *out->global_scale.  Each rank's codes and scales then equal
 *            those of the whole tensor quantised at once.
 *   Per block of 16: sb = E4M3_rn_satfinite(m / (6 S)), m the block amax;
 *   codes = E2M1_rn_satfinite(x * (1 / (E4M3(sb) * S))), all float32 ops
 *   rounded to nearest even; blocks whose E4M3(sb) * S is 0 get code 0.
 *   workspace: device, >= nvfp4_quantize_workspace_size() bytes, 16-byte
 *            aligned (required except with GIVEN_SCALE, where it may be NULL).
 * Requirements: rows >= 1, cols >= 64, cols % 64 == 0. */
NVFP4_API nvfp4_status nvfp4_quantize(const void* x, int32_t x_dtype, int64_t rows, int64_t cols, int64_t ld,
                            const nvfp4_tensor* out, int32_t flags, void* workspace,
                            size_t workspace_bytes, nvfp4_stream_t stream);

/* ----------------------------------------------------------------- GEMM -- */
/* Block-scaled FP4 x FP4 GEMM on the tcgen05 tensor cores (review page, paper
 * sec.6: the fused in_proj GEMM; the out_proj uses the same call):
 *   C[M x N] = S_A * S_B * sum_k (e2m1(A) e4m3(sfA))[m,k] (e2m1(B) e4m3(sfB))[n,k]
 * A: [M x K] NVFP4 (activations), B: [N x K] NVFP4 (weights, K-major rows).
 * C: device float32, row pitch ldc (ldc >= N, ldc % 4 == 0, C 16-byte aligned).
 * Requirements: K % 64 == 0, N % 4 == 0, A->cols == B->cols == K. */
NVFP4_API nvfp4_status w4a4_gemm(const nvfp4_tensor* A, const nvfp4_tensor* B, float* C, int64_t ldc,
                       nvfp4_stream_t stream);

/* ---------------------------------------------------------------- gates -- */
/* Gates, Eq.(1) (review page, paper sec.2), and per-head q/k L2 normalisation:
 *   proj: device float32 [n_tokens x ld_proj], the fused projection with
 *         column slices q [Hk*K] | k [Hk*K] | v [Hv*V] | z [Hv*V] | a [Hv] | b [Hv].
 *   q_hat, k_hat: device float32 [n_tokens x Hk x K]: x / sqrt(sum x^2 + 1e-6), computed
 *         as x * rsqrtf(sum x^2 + 1e-6) (the same in the scans' own normalisation).
 *   g:     device float32 [n_tokens x Hv]: -exp(A_log[h]) * softplus(a + dt_bias[h])
 *          (log of the decay alpha), softplus(u) = max(u,0) + log1p(exp(-|u|)).
 *   beta:  device float32 [n_tokens x Hv]: 1 / (1 + exp(-b)).
 *   A_log, dt_bias: device float32 [Hv]. */
NVFP4_API nvfp4_status gdn_gates(const float* proj, int64_t ld_proj, int64_t n_tokens, const gdn_dims* dims,
                       const float* A_log, const float* dt_bias, float* q_hat, float* k_hat,
                       float* g, float* beta, nvfp4_stream_t stream);

/* ----------------------------------------------------------------- scan -- */
/* Bytes of workspace gdn_scan needs for (B, T, dims, algo). */
NVFP4_API size_t gdn_scan_workspace_size(int32_t B, int64_t T, const gdn_dims* dims, int32_t algo);

/* Delta-rule recurrence, Eq.(2) (review page, background, paper sec.1), in
 * float32 with the state carried in float32:
 *   form GDN_FORM_PAGES:    S_t = a S + b k (v - S^T k)^T   (as the pages write it)
 *   form GDN_FORM_STANDARD: S_t = a S + b k (v - a S^T k)^T (decay inside the correction)
 *   o_t = scale * S_t^T q_t.
 * q_hat, k_hat: device [B x T x Hk x K]; v: device, token (b, t) row at
 * v + (b*T + t) * ld_v, head h at + h*V; g (log alpha), beta: device [B x T x Hv];
 * o: device [B x T x Hv x V]; state_in (NULL = zeros), state_out (NULL = not
 * written): device [B x Hv x K x V], 16-byte aligned.  state_in may equal state_out.
 * algo: AUTO (chunked for T > 1, recurrent for T == 1), RECURRENT (token by
 * token), CHUNKED (chunks of 64 tokens, WY/UT form).
 * workspace: device, >= gdn_scan_workspace_size(B, T, dims, algo) bytes. */
NVFP4_API nvfp4_status gdn_scan(const float* q_hat, const float* k_hat, const float* v, int64_t ld_v,
                      const float* g, const float* beta, int32_t B, int64_t T, const gdn_dims* dims,
                      float scale, int32_t form, int32_t algo, const float* state_in,
                      float* state_out, float* o, void* workspace, size_t workspace_bytes,
                      nvfp4_stream_t stream);

/* No counterpart in the paper: an allocation-free variant of gdn_scan for
 * callers that cannot allocate device memory themselves -- for example a
 * plugin inside a host framework that owns every allocation, or code running
 * while a stream is captured into a CUDA graph, where a cudaMalloc would break
 * the capture.  It runs the chunked algorithm (GDN_SCAN_CHUNKED) exactly as
 * gdn_scan does, with every argument meaning the same, but keeps the scratch in
 * a fixed array inside the library instead of a caller-provided workspace.
 * The array holds GDN_SCAN_NOALLOC_MAX_SCRATCH_BYTES bytes on each GPU that
 * uses it and is kept until the process exits.  It calls no cudaMalloc /
 * cudaFree and no allocating library routine.
 *   - Size limit: a problem whose scratch, gdn_scan_workspace_size(B, T, dims,
 *     GDN_SCAN_CHUNKED), exceeds the array is rejected with
 *     NVFP4_ERR_WORKSPACE before anything is launched (64 MiB covers, e.g.,
 *     B = 1, 32 value heads of 128 x 128, T <= 896).
 *   - First use: the first call on a device looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current and keeps it for
 *     the life of the process; make that first call before any stream capture
 *     begins.  A device reset (cudaDeviceReset, or the primary context being
 *     destroyed and re-created) invalidates the kept address: do not call this
 *     function on that device again in the same process.
 *   - Sharing: every call on a device uses the same array and leaves its
 *     contents behind (the chunk preparation overwrites all of it, nothing has
 *     to start at zero).  Calls whose executions overlap on the GPU -- on
 *     different streams, or from different host threads -- race on the array
 *     and give wrong results; serialise them. */
#define GDN_SCAN_NOALLOC_MAX_SCRATCH_BYTES ((size_t)64 << 20) /* 64 MiB */
NVFP4_API nvfp4_status gdn_scan_noalloc(const float* q_hat, const float* k_hat, const float* v, int64_t ld_v,
                                        const float* g, const float* beta, int32_t B, int64_t T,
                                        const gdn_dims* dims, float scale, int32_t form, const float* state_in,
                                        float* state_out, float* o, nvfp4_stream_t stream);

/* ------------------------------------------------------- state passing -- */
/* Joining spans of one sequence (for a sequence split across GPUs, or into
 * independent spans on one).  Eq.(2) (review page, background) is affine in
 * the state: a token maps S to A_t S + b_t k_t v_t^T with
 *   A_t = a_t I - b_t k_t k_t^T        (GDN_FORM_PAGES)
 *   A_t = a_t (I - b_t k_t k_t^T)      (GDN_FORM_STANDARD),
 * so a span started from S_in ends in P S_in + S_loc, P = A_T ... A_1, S_loc its
 * final state from a zero start, and its outputs are o_t = o_loc_t + S_in^T m_t
 * with m_t = scale P_t^T q_t (P_t = A_t ... A_1) and o_loc the zero-start
 * outputs.  The pages scan each window in one pass and say nothing about
 * splitting it; this is the plain reading of the recurrence's algebra.
 * Recipe: gdn_scan_span on every span (its zero-start scan o_loc, S_loc and
 * its maps P, m; the spans are independent), then for each span its initial
 * state S_in = gdn_state_combine over the maps of the spans before it, and
 * gdn_scan_correct(m, S_in, o_loc) for every span whose S_in is not zero. */

/* Bytes of workspace gdn_scan_transition needs. */
NVFP4_API size_t gdn_scan_transition_workspace_size(int32_t B, int64_t T, const gdn_dims* dims, int32_t algo);

/* The span map P and the query map m of B spans of T tokens each (the
 * recurrence run on v = 0 from S = I).  q_hat, k_hat, g, beta, scale, form,
 * algo: as for gdn_scan (the same inputs the span's gdn_scan takes; dims->V is
 * not used).  P: device float32 [B x Hv x K x K] (written); qmap: device float32
 * [B x T x Hv x K] (written).  P, qmap and the workspace must not overlap;
 * pointers 16-byte aligned; workspace 256-byte aligned, >=
 * gdn_scan_transition_workspace_size(B, T, dims, algo) bytes.  Costs one scan
 * of the span with V = K. */
NVFP4_API nvfp4_status gdn_scan_transition(const float* q_hat, const float* k_hat, const float* g,
                                           const float* beta, int32_t B, int64_t T, const gdn_dims* dims,
                                           float scale, int32_t form, int32_t algo, float* P, float* qmap,
                                           void* workspace, size_t workspace_bytes, nvfp4_stream_t stream);

/* Bytes of workspace gdn_scan_span needs. */
NVFP4_API size_t gdn_scan_span_workspace_size(int32_t B, int64_t T, const gdn_dims* dims, int32_t algo);

/* One call for a span's independent step: the zero-start scan (o as gdn_scan's
 * output, S_loc its final state) and the span maps (P, qmap as
 * gdn_scan_transition's).  With the chunked algorithm and K == V the two share
 * one chunk preparation (the maps' chunk records are the scan's with the
 * v-dependent part zeroed); otherwise it runs gdn_scan then
 * gdn_scan_transition.  Inputs as for gdn_scan; o [B x T x Hv x V], S_loc
 * [B x Hv x K x V], P [B x Hv x K x K], qmap [B x T x Hv x K], all device
 * float32, 16-byte aligned, not overlapping each other or the workspace
 * (256-byte aligned, >= gdn_scan_span_workspace_size bytes). */
NVFP4_API nvfp4_status gdn_scan_span(const float* q_hat, const float* k_hat, const float* v, int64_t ld_v,
                                     const float* g, const float* beta, int32_t B, int64_t T, const gdn_dims* dims,
                                     float scale, int32_t form, int32_t algo, float* o, float* S_loc, float* P,
                                     float* qmap, void* workspace, size_t workspace_bytes, nvfp4_stream_t stream);

/* The composition of m spans' maps in order, per (sequence, value head) i < n
 * (n = sequences x value heads):
 *   S = S_in[i];  S = P[j][i] S + S_loc[j][i] for j = 0 .. m-1;  S_out[i] = S.
 * P: device float32 [m x n x K x K]; S_loc: device float32 [m x n x K x V]
 * (NULL: zero); S_in, S_out: device float32 [n x K x V] (S_in NULL: zero).
 * S_out may be S_in, or the last S_loc (S_loc + (m-1) n K V), and must not
 * overlap P or any other part of S_loc.  m >= 1; K = 32, 64 or 128; V a
 * multiple of 32; P 16-byte aligned.  One launch for the whole chain. */
NVFP4_API nvfp4_status gdn_state_combine(const float* P, const float* S_loc, const float* S_in, float* S_out,
                                         int32_t m, int64_t n, int32_t K, int32_t V, nvfp4_stream_t stream);

/* o[b,t,h,:] += S_in[b,h]^T qmap[b,t,h,:]: the outputs of B spans of T tokens
 * that started from S_in instead of zero.  qmap: device float32 [B x T x Hv x K]
 * (from gdn_scan_transition); S_in: device float32 [B x Hv x K x V]; o: device
 * float32 [B x T x Hv x V], updated in place, not overlapping the others.  K, V
 * must be 64 or 128; pointers 16-byte aligned.  o_amax (device, nullable): the
 * maximum |o| after the update is folded into it with atomicMax on the float
 * bits (it must hold a non-negative float, e.g. 0, beforehand).  With the spans
 * on several GPUs, a max all-reduce of the word gives the whole sequence's
 * amax, from which S = amax / 2688 goes to nvfp4_quantize as a given scale. */
NVFP4_API nvfp4_status gdn_scan_correct(const float* qmap, const float* S_in, float* o, int32_t B, int64_t T,
                                        int32_t Hv, int32_t K, int32_t V, unsigned int* o_amax,
                                        nvfp4_stream_t stream);

/* ---------------------------------------------------------- output gate -- */
/* Optional output gate before out_proj.  The pages name z as one of the
 * projections that move the layer output y (review page, Table 3 discussion)
 * and keep the layer's norms unquantised ("Minima" section) but give no
 * formula; this library reads it as the usual gated RMSNorm, per token t and
 * value head h:
 *   out[t,h,:] = o[t,h,:] / sqrt(mean_i o[t,h,i]^2 + 1e-6) * w[:] * SiLU(z[t,h,:]),
 *   SiLU(z) = z / (1 + exp(-z)).
 * o, out: device float32 [n_tokens x Hv x V] (out may equal o); z: device, token
 * t's row at z + t * ld_z, head h at + h*V (the z slice of the fused projection);
 * w: device float32 [V], shared by the heads.  V must be 64 or 128; ld_z a
 * multiple of 4 and z 16-byte aligned.  amax_word (device, nullable): the
 * maximum |out| is folded into it with atomicMax on the float bits (it must hold
 * a non-negative float, e.g. 0, beforehand). */
NVFP4_API nvfp4_status gdn_output_gate(const float* o, const float* z, int64_t ld_z, const float* w,
                                       int64_t n_tokens, int32_t Hv, int32_t V, float* out,
                                       unsigned int* amax_word, nvfp4_stream_t stream);

/* ------------------------------------------------------ short convolution -- */
/* Optional short causal convolution on the q|k|v channels.  The pages list
 * convolutions among the layers kept unquantised (review page, "Minima"
 * section) and give nothing more; this library reads it as the usual Gated
 * DeltaNet short convolution, per sequence b, token t and channel c:
 *   out[b,t,c] = SiLU(sum_{j<W} w[c*W + j] * x[b, t-W+1+j, c]),
 * with inputs before token 0 taken from state_in[b, c, 0..W-2] (NULL: zeros).
 * x: device float32, token (b, t) row at x + (b*T + t)*ld_x, channels 0..C-1;
 * out: device float32, row at out + (b*T + t)*ld_out, must not overlap x;
 * w: device float32 [C x W], 2 <= W <= 4;
 * state_out (nullable): device float32 [B x C x (W-1)], the last W-1 inputs of
 * each sequence; it may equal state_in. */
NVFP4_API nvfp4_status gdn_short_conv(const float* x, int64_t ld_x, int32_t B, int64_t T, int32_t C, int32_t W,
                                      const float* w, const float* state_in, float* state_out, float* out,
                                      int64_t ld_out, nvfp4_stream_t stream);

/* ---------------------------------------------------------------- layer -- */
typedef struct {
    nvfp4_tensor w_in;    /* [N_in x hidden], N_in = 2*Hk*K + 2*Hv*V + 2*Hv, one global scale */
    nvfp4_tensor w_out;   /* [hidden x Hv*V] */
    const float* A_log;   /* device [Hv] */
    const float* dt_bias; /* device [Hv] */
    gdn_dims dims;
    int32_t hidden;
    const float* out_norm; /* device [V]: weight of the output gate (see
                              gdn_output_gate); NULL: o goes to out_proj as is */
    const float* conv_weight; /* device [(2*Hk*K + Hv*V) x conv_width]: short
                                 convolution on q|k|v (see gdn_short_conv); NULL: none */
    int32_t conv_width;       /* 2..4 when conv_weight is set */
} gdn_layer_weights;

/* Byte offsets of the intermediates gdn_layer_forward leaves in its
 * workspace (valid after the stream reaches the call). */
typedef struct {
    size_t x_codes, x_sf, x_scale; /* quantised input */
    size_t proj;                   /* float32 [B*T x N_in] fused projection */
    size_t q_hat, k_hat, g, beta;  /* g, beta: the gates; q_hat, k_hat: room for gdn_gates'
                                      normalised q, k (the layer's scans normalise q and k
                                      themselves and leave these two regions unwritten) */
    size_t o;                      /* float32 [B*T x Hv*V] scan output */
    size_t o_gated;                /* float32 [B*T x Hv*V] gated output (an empty
                                      region when out_norm is NULL) */
    size_t qkv_conv;               /* float32 [B*T x (2*Hk*K + Hv*V)] convolved q|k|v
                                      (an empty region when conv_weight is NULL) */
    size_t o_codes, o_sf, o_scale; /* quantised scan output */
    size_t quant_ws;               /* quantiser scratch */
    size_t scan_ws;                /* scan scratch */
    size_t total;                  /* bytes required */
} gdn_layer_ws_layout;

NVFP4_API nvfp4_status gdn_layer_workspace_layout(const gdn_layer_weights* w, int32_t B, int64_t T,
                                        gdn_layer_ws_layout* out /* host */);

/* One GDN layer forward under NVFP4 W4A4 (the four steps above, then the
 * NVFP4 out_proj; with w->conv_weight set, q|k|v first pass through the short
 * convolution; with w->out_norm set, out_proj reads the output gate's G
 * instead of o):
 *   x_bf16: device bf16 [B*T x hidden]; y: device float32 [B*T x hidden].
 *   state_in (NULL = zeros) / state_out (NULL = not written): device float32
 *   [B x Hv x K x V], 16-byte aligned.  form: GDN_FORM_PAGES or GDN_FORM_STANDARD.
 *   workspace: device, >= the layout's `total` bytes, 256-byte aligned. */
NVFP4_API nvfp4_status gdn_layer_forward(const gdn_layer_weights* w, const void* x_bf16, int32_t B, int64_t T,
                               float* y, const float* state_in, float* state_out, int32_t form,
                               void* workspace, size_t workspace_bytes, nvfp4_stream_t stream);

/* gdn_layer_forward with the short convolution's carried inputs (used only when
 * w->conv_weight is set): conv_state_in (NULL: zeros) and conv_state_out (NULL:
 * not written), device float32 [B x (2*Hk*K + Hv*V) x (conv_width-1)]; they may
 * be the same buffer.  gdn_layer_forward is this call with both NULL. */
NVFP4_API nvfp4_status gdn_layer_forward_stateful(const gdn_layer_weights* w, const void* x_bf16, int32_t B,
                                                  int64_t T, float* y, const float* state_in, float* state_out,
                                                  const float* conv_state_in, float* conv_state_out, int32_t form,
                                                  void* workspace, size_t workspace_bytes, nvfp4_stream_t stream);

/* gdn_layer_forward_stateful that also records seven caller-created CUDA
 * events (cudaEvent_t, passed as void*) on the stream, for per-stage timing of
 * the layer's own launches: events[i] before stage i (0 quantise x, 1 in_proj,
 * 2 gates and the optional short convolution, 3 scan, 4 the optional output gate
 * and quantise o, 5 out_proj) and events[6] after out_proj.  The launches are
 * those of gdn_layer_forward_stateful; null events or a null handle: status 1. */
NVFP4_API nvfp4_status gdn_layer_forward_timed(const gdn_layer_weights* w, const void* x_bf16, int32_t B, int64_t T,
                                               float* y, const float* state_in, float* state_out,
                                               const float* conv_state_in, float* conv_state_out, int32_t form,
                                               void* workspace, size_t workspace_bytes, nvfp4_stream_t stream,
                                               void* const* events);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_GDN_H */
