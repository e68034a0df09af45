"""The studies' steps restated with the oracle (float64 numpy), so that the
study code of nvfp4_w4a4_gated_b200.studies runs on CPU on tiny shapes."""
import numpy as np

import oracle


class OracleBackend:
    def upload(self, a):
        return np.array(a, dtype=np.float64)

    def host(self, t):
        return np.asarray(t, dtype=np.float64)

    def rel(self, a, b):
        return float(np.linalg.norm(a - b) / np.linalg.norm(b))

    def norm(self, a):
        return float(np.linalg.norm(a))

    def cat_rows(self, parts):
        return np.concatenate(parts, axis=0)

    def copy(self, a):
        return np.array(a, copy=True)

    def assign_cols(self, dst, c0, c1, src):
        dst[:, c0:c1] = src[:, c0:c1]

    def noise_factors(self, seed, n_rows, n_cols, sigma):
        g = np.random.Generator(np.random.PCG64(seed))
        return (1.0 + sigma * g.standard_normal((n_rows, n_cols))).astype(np.float32).astype(np.float64)

    def scale_cols(self, dst, c0, c1, factor):
        dst[:, c0:c1] *= factor

    def add(self, a, b):
        return a + b

    def matmul_nt(self, x, W):
        return oracle.gemm_nt(x, W)

    def quantize(self, W):
        return oracle.quantize(np.asarray(W, np.float32))

    def w4a4(self, x, Wq):
        return oracle.w4a4_gemm(oracle.quantize(np.asarray(x, np.float32)), Wq)

    def gates(self, P, dims, A_log, dt_bias):
        q, k, v, _, a, b = oracle.split_projection(P, dims.Hk, dims.Hv, dims.K, dims.V)
        g, beta = oracle.gates(a, b, A_log, dt_bias)
        n = P.shape[0]
        return (oracle.l2norm(q.reshape(n, dims.Hk, dims.K)), oracle.l2norm(k.reshape(n, dims.Hk, dims.K)),
                np.ascontiguousarray(v), g, beta)

    def gate_exp(self, g):
        return 1.0 - np.exp(g)

    def log_mul(self, g, factor):
        return g + np.log(factor)

    def mul(self, a, factor):
        return a * factor

    def scan(self, q_hat, k_hat, v, g, beta, B, T, dims, S0=None, form=oracle.FORM_PAGES):
        o, S = oracle.scan(q_hat.reshape(B, T, dims.Hk, dims.K), k_hat.reshape(B, T, dims.Hk, dims.K),
                           v.reshape(B, T, dims.Hv, dims.V), g.reshape(B, T, dims.Hv), beta.reshape(B, T, dims.Hv),
                           form=form, S0=S0)
        return o.reshape(B * T, dims.Hv, dims.V), S

    def output_gate(self, o, z, w):
        n, Hv, V = o.shape
        # the layer's out_proj reads float32 o
        return oracle.output_gate(o.astype(np.float32), z.reshape(n, Hv, V), w)

    def zeros_like(self, a):
        return np.zeros_like(a)
