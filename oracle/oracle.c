/*
 * oracle.c -- plain, slow, CPU reference for the NVFP4 W4A4 Gated DeltaNet layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the package's smoke check and the timed CPU
 * baseline in the benchmark use it.  It shares no source with the CUDA library.
 *
 * Sources (web pages on "Why Gated DeltaNet Survives 4-Bit Quantization:
 * NVFP4 W4A4 for the Recurrent Half of a Hybrid 27B LLM"):
 *   [R]  the jaehun.me review of the paper (background section citing paper
 *        sec.1 for the NVFP4 format and Eq.(2) for the recurrence; sec.2 /
 *        Eq.(1) for the gates; sec.5.1 for block scaling; sec.5.3 for the
 *        delta-rule overwrite; sec.6 for global-scale harmonisation).
 *   [A]  the paper's abstract (transistor.fm page): fused-GEMM global-scale
 *        mismatch and its repair.
 *   [S]  the SoloQ summary page (onedev.kr): NVFP4 scales computed dynamically
 *        from the tensor itself.
 *
 * Precision: the quantiser is an exact float32 (IEEE, round-to-nearest-even)
 * op sequence, because its outputs are integer codes that the GPU must match
 * bit for bit.  Everything else is float64.
 *
 * Readings of points the pages leave open (each mirrored, independently, by
 * the CUDA library):
 *   Q1 global scale S = fl32(amax / 2688), 2688 = 6 * 448, S is the dequant
 *      multiplier; S := 1 when amax < 2^-100 (that includes amax == 0).
 *   Q2 block scale sb = E4M3_rne_satfinite(fl32(m / fl32(6 * S))), m = block amax.
 *   Q3 element code = E2M1_rne_satfinite(fl32(x * fl32(1 / fl32(E4M3(sb) * S)))),
 *      sign kept (so -0 encodes as 0x8); if fl32(E4M3(sb) * S) == 0 the block's
 *      codes are all 0x0.
 *   Q4 packing: element 2i in the low nibble, 2i+1 in the high nibble; code bits
 *      s|e1 e0|m.
 *   G1 softplus(u) = max(u,0) + log1p(exp(-|u|)) (no threshold switch).
 *   G2 q/k normalisation x / sqrt(sum x^2 + 1e-6) per head.
 *   S1 form PAGES:    S_t = a S + b k (v - S^T k)^T         (the pages' Eq.(2))
 *      form STANDARD: S_t = a S + b k (v - a S^T k)^T       (decay inside)
 *   S2 value head h reads key head floor(h * Hk / Hv); zero initial state.
 *   O1 output gate (optional; [R] names the z projection as one that moves the
 *      output y, Table 3 discussion, and keeps the norms unquantised, "Minima"
 *      section, but gives no formula): per token and value head,
 *      G = o / sqrt(mean(o^2) + 1e-6) * w * z * sigmoid(z), w a learned weight
 *      of V entries shared by the heads; out_proj then reads G instead of o.
 *   P1 state passing (the sequence-sharded scan): the pages run the recurrence
 *      over windows of up to 32K tokens ([R] sec.5.3) in one pass and say
 *      nothing about splitting it; here a sequence is split into spans that
 *      are joined through the affinity of Eq.(2) in the state
 *      (orc_scan_transition).
 *   C1 short convolution (optional; [R] lists convolutions among the layers kept
 *      unquantised, "Minima" section, and gives nothing else): per channel c of
 *      the q|k|v slices, a causal depthwise convolution of width W followed by
 *      SiLU, out_t[c] = SiLU(sum_j w[c][j] x_{t-W+1+j}[c]); inputs before the
 *      first token come from a carried state (the previous W-1 inputs, zero when
 *      absent), and the new state is the last W-1 inputs.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <fenv.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* Number formats ([R] background / paper sec.1: E2M1 values, one E4M3 scale */
/* per 16-element block, one FP32 scale per tensor).                         */
/* ------------------------------------------------------------------------ */

/* E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; no inf/nan.
 * Magnitudes by code 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
ORC_EXPORT double orc_e2m1_decode(uint8_t code) {
    int e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return (code & 8) ? -mag : mag;
}

/* Round |y| to the E2M1 grid, ties to even mantissa, saturating at 6.
 * The spacing is 0.5 below 2, 1 in [2,4), 2 from 4 on; rounding to an even
 * multiple of the spacing is rounding to an even mantissa. */
ORC_EXPORT uint8_t orc_e2m1_encode(float y) {
    uint8_t sign = signbit(y) ? 8 : 0;
    double a = fabs((double)y);
    double step = (a < 2.0) ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
    double r = nearbyint(a / step) * step;       /* default rounding mode: ties to even */
    if (r > 6.0) r = 6.0;
    uint8_t code;
    if (r < 1.0) code = (uint8_t)(r * 2.0);      /* 0 -> 0, 0.5 -> 1 */
    else {
        int e = ilogb(r);                       /* 0,1,2 */
        double m = r / ldexp(1.0, e) - 1.0;     /* 0 or 0.5 */
        code = (uint8_t)(((e + 1) << 1) | (m > 0.0 ? 1 : 0));
    }
    return sign | code;
}

/* E4M3 ("FN": no inf, max 448, 0x7F / 0xFF are NaN): bias 7, 3 mantissa bits,
 * subnormal step 2^-9. */
ORC_EXPORT double orc_e4m3_decode(uint8_t b) {
    int e = (b >> 3) & 15, m = b & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return (b & 0x80) ? -mag : mag;
}

/* Non-negative finite input only (block scales are magnitudes).
 * Round to nearest, ties to even, saturate at 448. */
ORC_EXPORT uint8_t orc_e4m3_encode(float s) {
    double a = (double)s;
    if (!(a > 0.0)) return 0;
    if (a >= 448.0) return 0x7E;
    int e = ilogb(a);
    if (e < -6) e = -6;                          /* subnormal range shares the 2^-9 step */
    double step = ldexp(1.0, e - 3);
    double r = nearbyint(a / step) * step;
    if (r > 448.0) r = 448.0;
    if (r == 0.0) return 0;
    if (r < ldexp(1.0, -6)) return (uint8_t)(r / ldexp(1.0, -9));
    int er = ilogb(r);
    int m = (int)((r / ldexp(1.0, er) - 1.0) * 8.0);
    return (uint8_t)(((er + 7) << 3) | m);
}

/* ------------------------------------------------------------------------ */
/* Quantiser (readings Q1-Q4).                                               */
/* ------------------------------------------------------------------------ */

/* Per-tensor scale from the tensor's amax ([R] background; [S]: scales are
 * derived from the tensor itself at run time). */
ORC_EXPORT float orc_global_scale(const float* x, int64_t n) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    if (amax < 0x1p-100f) return 1.0f;
    volatile float den = 2688.0f;
    return amax / den;
}

/* Quantise x [rows x cols] (row-major, cols % 16 == 0) under global scale S.
 * codes: [rows x cols/2] packed nibbles; sf: [rows x cols/16] linear layout. */
ORC_EXPORT void orc_quantize(const float* x, int64_t rows, int64_t cols, float S,
                             uint8_t* codes, uint8_t* sf) {
    const int64_t nb = cols / 16;
    volatile float six = 6.0f, one = 1.0f;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* blk = x + r * cols + b * 16;
            float m = 0.0f;
            for (int i = 0; i < 16; ++i) { float a = fabsf(blk[i]); if (a > m) m = a; }
            volatile float d = six * S;
            volatile float s_f = m / d;
            uint8_t sb = orc_e4m3_encode(s_f);
            volatile float dec = (float)orc_e4m3_decode(sb) * S;
            sf[r * nb + b] = sb;
            uint8_t* cb = codes + r * (cols / 2) + b * 8;
            if (dec == 0.0f) { memset(cb, 0, 8); continue; }
            volatile float inv = one / dec;
            for (int i = 0; i < 8; ++i) {
                volatile float y0 = blk[2 * i] * inv;
                volatile float y1 = blk[2 * i + 1] * inv;
                cb[i] = (uint8_t)(orc_e2m1_encode(y0) | (orc_e2m1_encode(y1) << 4));
            }
        }
    }
}

/* Dequantise to float64: x_hat = e2m1(code) * e4m3(sb) * S (every factor exact
 * in double). */
ORC_EXPORT void orc_dequantize(const uint8_t* codes, const uint8_t* sf, float S,
                               int64_t rows, int64_t cols, double* out) {
    const int64_t nb = cols / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            uint8_t code = (c & 1) ? (byte >> 4) : (byte & 15);
            out[r * cols + c] = orc_e2m1_decode(code) * orc_e4m3_decode(sf[r * nb + c / 16]) * (double)S;
        }
}

/* Scale-factor layout read by the block-scaled tensor-core MMA: 128-row x
 * 4-block atoms of 512 bytes, atoms ordered (row block, k block) with k
 * fastest; inside an atom the byte for (row r, block j) sits at
 * (r % 32) * 16 + (r / 32) * 4 + j.  Rows are padded to a multiple of 128
 * (pad bytes 0).  A pure permutation of the linear layout. */
ORC_EXPORT void orc_sf_linear_to_mma(const uint8_t* sf, int64_t rows, int64_t cols, uint8_t* out) {
    const int64_t nb = cols / 16, nkb = nb / 4;
    const int64_t prow = (rows + 127) / 128 * 128;
    memset(out, 0, (size_t)(prow * nb));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            int64_t atom = (r / 128) * nkb + b / 4;
            int64_t rr = r % 128;
            out[atom * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (b % 4)] = sf[r * nb + b];
        }
}

/* ------------------------------------------------------------------------ */
/* GEMM: C[M x N] = A[M x K] * B[N x K]^T in float64 (a textbook triple loop). */
/* ------------------------------------------------------------------------ */
ORC_EXPORT void orc_gemm_nt(const double* A, const double* B, int64_t M, int64_t N, int64_t K,
                            double* C) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            const double* a = A + i * K;
            const double* b = B + j * K;
            for (int64_t k = 0; k < K; ++k) acc += a[k] * b[k];
            C[i * N + j] = acc;
        }
}

/* ------------------------------------------------------------------------ */
/* Gates ([R] sec.2, Eq.(1)) and q/k normalisation (reading G2).             */
/* ------------------------------------------------------------------------ */
ORC_EXPORT double orc_softplus(double u) { return fmax(u, 0.0) + log1p(exp(-fabs(u))); }

/* a, b: [n x Hv] gate pre-activations.  Outputs g = log(alpha) and beta. */
ORC_EXPORT void orc_gates(const double* a, const double* b, const double* A_log,
                          const double* dt_bias, int64_t n, int32_t Hv, double* g, double* beta) {
    for (int64_t t = 0; t < n; ++t)
        for (int32_t h = 0; h < Hv; ++h) {
            int64_t i = t * Hv + h;
            g[i] = -exp(A_log[h]) * orc_softplus(a[i] + dt_bias[h]);
            beta[i] = 1.0 / (1.0 + exp(-b[i]));
        }
}

/* x: [n x H x D] rows of length D normalised in place to unit L2 norm. */
ORC_EXPORT void orc_l2norm(double* x, int64_t nrows, int32_t D, double eps) {
    for (int64_t r = 0; r < nrows; ++r) {
        double s = 0.0;
        for (int32_t i = 0; i < D; ++i) s += x[r * D + i] * x[r * D + i];
        double inv = 1.0 / sqrt(s + eps);
        for (int32_t i = 0; i < D; ++i) x[r * D + i] *= inv;
    }
}

/* Output gate (reading O1).  o, z, out: [n x Hv x V]; w: [V]. */
ORC_EXPORT void orc_output_gate(const double* o, const double* z, const double* w, int64_t n, int32_t Hv,
                                int32_t V, double eps, double* out) {
    for (int64_t r = 0; r < n * Hv; ++r) {
        const double* orow = o + r * V;
        const double* zrow = z + r * V;
        double ms = 0.0;
        for (int32_t i = 0; i < V; ++i) ms += orow[i] * orow[i];
        ms /= V;
        double inv_rms = 1.0 / sqrt(ms + eps);
        for (int32_t i = 0; i < V; ++i) {
            double silu = zrow[i] / (1.0 + exp(-zrow[i]));
            out[r * V + i] = orow[i] * inv_rms * w[i] * silu;
        }
    }
}

/* Short causal convolution (reading C1).  x: token (b, t) row at x + (b*T + t)*ldx,
 * channels 0..C-1; w: [C x W]; state_in, state_out: [B x C x (W-1)] (NULL: zeros /
 * not written); out: [B*T x C].  silu = 0 returns the pre-activation. */
ORC_EXPORT void orc_short_conv(const double* x, int64_t ldx, int32_t B, int64_t T, int32_t C, int32_t W,
                               const double* w, const double* state_in, double* state_out, double* out,
                               int32_t silu) {
    for (int32_t b = 0; b < B; ++b)
        for (int32_t c = 0; c < C; ++c) {
            /* input at token index u (u may be negative: from the state) */
            for (int64_t t = 0; t < T; ++t) {
                double acc = 0.0;
                for (int32_t j = 0; j < W; ++j) {
                    int64_t u = t - (W - 1) + j;
                    double xv;
                    if (u >= 0)
                        xv = x[(b * T + u) * ldx + c];
                    else
                        xv = state_in ? state_in[((int64_t)b * C + c) * (W - 1) + (u + (W - 1))] : 0.0;
                    acc += w[(int64_t)c * W + j] * xv;
                }
                out[(b * T + t) * C + c] = silu ? acc / (1.0 + exp(-acc)) : acc;
            }
            if (state_out)
                for (int32_t i = 0; i < W - 1; ++i) {
                    int64_t u = T - (W - 1) + i;
                    double xv;
                    if (u >= 0)
                        xv = x[(b * T + u) * ldx + c];
                    else
                        xv = state_in ? state_in[((int64_t)b * C + c) * (W - 1) + (u + (W - 1))] : 0.0;
                    state_out[((int64_t)b * C + c) * (W - 1) + i] = xv;
                }
        }
}

/* ------------------------------------------------------------------------ */
/* Delta-rule recurrence ([R] background, Eq.(2)), token by token.           */
/*   q, k: [B, T, Hk, K]; v, o: [B, T, Hv, V]; g, beta: [B, T, Hv];           */
/*   S0, S: [B, Hv, K, V] (S0 may be NULL = zeros).                           */
/*   form 0 = PAGES, 1 = STANDARD (reading S1).                               */
/* ------------------------------------------------------------------------ */
ORC_EXPORT void orc_scan(const double* q, const double* k, const double* v, const double* g,
                         const double* beta, int32_t B, int64_t T, int32_t Hk, int32_t Hv,
                         int32_t K, int32_t V, double scale, int32_t form, const double* S0,
                         double* S, double* o) {
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t bb = 0; bb < B; ++bb)
        for (int32_t h = 0; h < Hv; ++h) {
            const int32_t hk = (int32_t)(((int64_t)h * Hk) / Hv);
            double* St = S + ((int64_t)bb * Hv + h) * K * V;
            if (S0) memcpy(St, S0 + ((int64_t)bb * Hv + h) * K * V, sizeof(double) * K * V);
            else memset(St, 0, sizeof(double) * K * V);
            double* pred = (double*)malloc(sizeof(double) * V);
            for (int64_t t = 0; t < T; ++t) {
                const double* kt = k + (((int64_t)bb * T + t) * Hk + hk) * K;
                const double* qt = q + (((int64_t)bb * T + t) * Hk + hk) * K;
                const double* vt = v + (((int64_t)bb * T + t) * Hv + h) * V;
                double* ot = o + (((int64_t)bb * T + t) * Hv + h) * V;
                const double alpha = exp(g[((int64_t)bb * T + t) * Hv + h]);
                const double bt = beta[((int64_t)bb * T + t) * Hv + h];
                /* prediction S_{t-1}^T k_t (decayed first in the STANDARD form) */
                for (int32_t j = 0; j < V; ++j) {
                    double s = 0.0;
                    for (int32_t i = 0; i < K; ++i) s += St[(int64_t)i * V + j] * kt[i];
                    pred[j] = (form == 1) ? alpha * s : s;
                }
                for (int32_t i = 0; i < K; ++i)
                    for (int32_t j = 0; j < V; ++j)
                        St[(int64_t)i * V + j] = alpha * St[(int64_t)i * V + j] + bt * kt[i] * (vt[j] - pred[j]);
                for (int32_t j = 0; j < V; ++j) {
                    double s = 0.0;
                    for (int32_t i = 0; i < K; ++i) s += St[(int64_t)i * V + j] * qt[i];
                    ot[j] = s * scale;
                }
            }
            free(pred);
        }
}

/* Chunked form of the same recurrence (used only to pin the derivation that
 * the GPU's chunked kernel follows; tiny shapes).  Within a chunk of C tokens
 * with G_t = sum_{j<=t} g_j:
 *   u_t + b_t sum_{i<t} e^{G_{t-1}-G_i} (k_t.k_i) u_i = beta_t v_t - b_t e^{G_{t-1}} S0^T k_t
 *   (b_t = beta_t for PAGES, alpha_t beta_t for STANDARD)
 *   o_t   = scale * (e^{G_t} S0^T q_t + sum_{i<=t} e^{G_t-G_i} (q_t.k_i) u_i)
 *   S_C   = e^{G_C} S0 + sum_i e^{G_C-G_i} k_i u_i^T
 * Solved by forward substitution, one chunk at a time. */
ORC_EXPORT void orc_scan_chunked(const double* q, const double* k, const double* v, const double* g,
                                 const double* beta, int32_t B, int64_t T, int32_t Hk, int32_t Hv,
                                 int32_t K, int32_t V, double scale, int32_t form, int32_t C,
                                 const double* S0, double* S, double* o) {
    for (int32_t bb = 0; bb < B; ++bb)
        for (int32_t h = 0; h < Hv; ++h) {
            const int32_t hk = (int32_t)(((int64_t)h * Hk) / Hv);
            double* St = S + ((int64_t)bb * Hv + h) * K * V;
            if (S0) memcpy(St, S0 + ((int64_t)bb * Hv + h) * K * V, sizeof(double) * K * V);
            else memset(St, 0, sizeof(double) * K * V);
            double* G = (double*)malloc(sizeof(double) * (C + 1));
            double* U = (double*)malloc(sizeof(double) * C * V);
            double* Sn = (double*)malloc(sizeof(double) * K * V);
            for (int64_t t0 = 0; t0 < T; t0 += C) {
                const int32_t n = (int32_t)((T - t0) < C ? (T - t0) : C);
                G[0] = 0.0;
                for (int32_t t = 1; t <= n; ++t) G[t] = G[t - 1] + g[((int64_t)bb * T + t0 + t - 1) * Hv + h];
#define KV(t) (k + (((int64_t)bb * T + t0 + (t) - 1) * Hk + hk) * K)
#define QV(t) (q + (((int64_t)bb * T + t0 + (t) - 1) * Hk + hk) * K)
#define VV(t) (v + (((int64_t)bb * T + t0 + (t) - 1) * Hv + h) * V)
                for (int32_t t = 1; t <= n; ++t) {
                    const double bt = beta[((int64_t)bb * T + t0 + t - 1) * Hv + h];
                    const double at = exp(G[t] - G[t - 1]);
                    const double bk = (form == 1) ? at * bt : bt;
                    const double* kt = KV(t);
                    for (int32_t j = 0; j < V; ++j) {
                        double s0k = 0.0;
                        for (int32_t i = 0; i < K; ++i) s0k += St[(int64_t)i * V + j] * kt[i];
                        double rhs = bt * VV(t)[j] - bk * exp(G[t - 1]) * s0k;
                        for (int32_t i = 1; i < t; ++i) {
                            double kk = 0.0;
                            for (int32_t d = 0; d < K; ++d) kk += kt[d] * KV(i)[d];
                            rhs -= bk * exp(G[t - 1] - G[i]) * kk * U[(int64_t)(i - 1) * V + j];
                        }
                        U[(int64_t)(t - 1) * V + j] = rhs;
                    }
                }
                for (int32_t t = 1; t <= n; ++t) {
                    const double* qt = QV(t);
                    double* ot = o + (((int64_t)bb * T + t0 + t - 1) * Hv + h) * V;
                    for (int32_t j = 0; j < V; ++j) {
                        double s = 0.0;
                        for (int32_t i = 0; i < K; ++i) s += St[(int64_t)i * V + j] * qt[i];
                        s *= exp(G[t]);
                        for (int32_t i = 1; i <= t; ++i) {
                            double qk = 0.0;
                            for (int32_t d = 0; d < K; ++d) qk += qt[d] * KV(i)[d];
                            s += exp(G[t] - G[i]) * qk * U[(int64_t)(i - 1) * V + j];
                        }
                        ot[j] = s * scale;
                    }
                }
                for (int32_t i = 0; i < K; ++i)
                    for (int32_t j = 0; j < V; ++j) {
                        double s = exp(G[n]) * St[(int64_t)i * V + j];
                        for (int32_t t = 1; t <= n; ++t) s += exp(G[n] - G[t]) * KV(t)[i] * U[(int64_t)(t - 1) * V + j];
                        Sn[(int64_t)i * V + j] = s;
                    }
                memcpy(St, Sn, sizeof(double) * K * V);
#undef KV
#undef QV
#undef VV
            }
            free(G); free(U); free(Sn);
        }
}

/* ------------------------------------------------------------------------ */
/* State passing (reading P1).  Eq.(2) is affine in the state: with           */
/*   A_t = a_t I - b_t k_t k_t^T          (form PAGES)                        */
/*   A_t = a_t (I - b_t k_t k_t^T)        (form STANDARD)                     */
/* one token maps S to A_t S + b_t k_t v_t^T, so a span of tokens maps an     */
/* initial state S_in to P S_in + S_loc, with P = A_T ... A_1 and S_loc the   */
/* span's final state from a zero start, and each output of the span gains   */
/* S_in^T (scale P_t^T q_t), P_t = A_t ... A_1.  This function forms P and    */
/* the query map m_t = scale P_t^T q_t straight from that product, one token  */
/* at a time: A_t P = a_t P - b_t k_t (k_t^T P) for PAGES and                 */
/* a_t (P - b_t k_t (k_t^T P)) for STANDARD.                                  */
/*   q, k: [B, T, Hk, K]; g, beta: [B, T, Hv]; P: [B, Hv, K, K];              */
/*   qmap: [B, T, Hv, K].                                                     */
/* ------------------------------------------------------------------------ */
ORC_EXPORT void orc_scan_transition(const double* q, const double* k, const double* g, const double* beta,
                                    int32_t B, int64_t T, int32_t Hk, int32_t Hv, int32_t K, double scale,
                                    int32_t form, double* P, double* qmap) {
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t bb = 0; bb < B; ++bb)
        for (int32_t h = 0; h < Hv; ++h) {
            const int32_t hk = (int32_t)(((int64_t)h * Hk) / Hv);
            double* Pt = P + ((int64_t)bb * Hv + h) * K * K;
            for (int32_t i = 0; i < K; ++i)
                for (int32_t j = 0; j < K; ++j) Pt[(int64_t)i * K + j] = (i == j) ? 1.0 : 0.0;
            double* kP = (double*)malloc(sizeof(double) * K);
            for (int64_t t = 0; t < T; ++t) {
                const double* kt = k + (((int64_t)bb * T + t) * Hk + hk) * K;
                const double* qt = q + (((int64_t)bb * T + t) * Hk + hk) * K;
                const double alpha = exp(g[((int64_t)bb * T + t) * Hv + h]);
                const double bt = beta[((int64_t)bb * T + t) * Hv + h];
                for (int32_t j = 0; j < K; ++j) {           /* k_t^T P, a row vector */
                    double s = 0.0;
                    for (int32_t i = 0; i < K; ++i) s += kt[i] * Pt[(int64_t)i * K + j];
                    kP[j] = s;
                }
                for (int32_t i = 0; i < K; ++i)
                    for (int32_t j = 0; j < K; ++j) {
                        const double rank1 = bt * kt[i] * kP[j];
                        double* e = &Pt[(int64_t)i * K + j];
                        *e = (form == 1) ? alpha * (*e - rank1) : alpha * (*e) - rank1;
                    }
                double* mt = qmap + (((int64_t)bb * T + t) * Hv + h) * K;
                for (int32_t j = 0; j < K; ++j) {           /* scale P_t^T q_t */
                    double s = 0.0;
                    for (int32_t i = 0; i < K; ++i) s += Pt[(int64_t)i * K + j] * qt[i];
                    mt[j] = s * scale;
                }
            }
            free(kP);
        }
}

ORC_EXPORT int32_t orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
