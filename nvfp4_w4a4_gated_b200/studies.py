"""Mechanism studies of the review page of "Why Gated DeltaNet Survives 4-Bit
Quantization" (paper sec.5.2 Table 3; sec.5.3 Fig. 1 and Table 6), run on
synthetic inputs through this library's kernels.

1. Per-projection sensitivity replay (sec.5.2, Table 3): the layer is run with
   one projection at a time under NVFP4 W4A4 (q|k|v, z, a, b, out) and the
   rest unquantised; for each, the projection's own error, the movement of the
   layer output y and of the final state, and, for the gate projections, the
   error that reaches 1 - alpha and beta.  Then all at once, beside the
   root-sum-square of the single-projection y errors (the pages find the two
   equal: the errors are independent).
2. Lockstep trajectories (sec.5.3, Fig. 1a): one clean recurrence and eleven
   perturbed ones on the same input, carried side by side in float32 state;
   the relative state error relS_t = |S'_t - S_t| / |S_t| at checkpoints.  The
   first perturbed trajectory is the W4A4 layer's; the other ten add seeded
   Gaussian noise to each projection at that projection's measured W4A4 error.
   Then a 1% state impulse injected at t = 1024 and the number of steps until
   its size falls to 1/e and 1/10 (Fig. 1b), beside the horizon 1/(1 - alpha)
   the decay gates alone imply.
3. Gate-noise table (sec.5.3, Table 6): the state error after multiplicative
   noise on alpha (0.1%), after quantising only the a projection, and after
   multiplicative noise on beta (1%).

The pages measure these on captured activations of a trained 27B model; with
random weights the numbers are context, not a reproduction.  Reading of the
pages used here: "perturbed trajectories" are read as projections carrying
W4A4-sized errors (the pages do not say how the eleven differ); the layer
output is taken through the output gate with a unit weight (reading O1), since
z moves y only through it.

Every product and the recurrence run in the library's kernels (W4A4 GEMM,
quantiser, gates, chunked scan, output gate); the unquantised reference
products are float32 matmuls (TF32 off) on the GPU, the reference every W4A4
error is measured against.  ``backend`` lets the same study code run on other
implementations of the steps (the CPU tests use the oracle's).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

from . import (FORM_PAGES, SCAN_CHUNKED, SCAN_RECURRENT, GdnDims, gdn_gates, gdn_output_gate, gdn_scan,
               nvfp4_quantize, w4a4_gemm)


# ------------------------------------------------------------------ backend --
class CudaBackend:
    """The studies' steps on the GPU: this library's kernels for the W4A4 path,
    the gates, the scan and the output gate; float32 matmuls for the
    unquantised reference products."""

    def __init__(self, device="cuda", device_noise: bool = False):
        self.dev = torch.device(device)
        self.device_noise = device_noise

    def noise_factors(self, seed, n_rows, n_cols, sigma):
        """1 + sigma * N(0, 1), seeded: drawn on the host (numpy PCG64, the same
        numbers as the oracle backend's) or, with device_noise, on the GPU."""
        if not self.device_noise:
            return self.upload(_noise_factors(seed, n_rows, n_cols, sigma))
        gen = torch.Generator(device=self.dev)
        gen.manual_seed(seed)
        return 1.0 + sigma * torch.randn((n_rows, n_cols), generator=gen, device=self.dev)

    # arrays
    def upload(self, a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(self.dev)

    def host(self, t):
        return t.detach().double().cpu().numpy()

    def rel(self, a, b) -> float:
        return float(torch.linalg.vector_norm((a - b).double()) / torch.linalg.vector_norm(b.double()))

    def norm(self, a) -> float:
        return float(torch.linalg.vector_norm(a.double()))

    def cat_rows(self, parts):
        return torch.cat(parts, dim=0)

    def copy(self, a):
        return a.clone()

    def assign_cols(self, dst, c0, c1, src):
        dst[:, c0:c1] = src[:, c0:c1]

    def scale_cols(self, dst, c0, c1, factor):
        """dst[:, c0:c1] *= factor (that block's shape)."""
        dst[:, c0:c1] *= factor

    def add(self, a, b):
        return a + b

    # steps
    def matmul_nt(self, x, W):
        prev = torch.backends.cuda.matmul.allow_tf32
        torch.backends.cuda.matmul.allow_tf32 = False
        try:
            return x @ W.T
        finally:
            torch.backends.cuda.matmul.allow_tf32 = prev

    def quantize(self, W):
        return nvfp4_quantize(W)

    def w4a4(self, x, Wq):
        return w4a4_gemm(nvfp4_quantize(x.contiguous()), Wq)

    def gates(self, P, dims, A_log, dt_bias):
        q_hat, k_hat, g, beta = gdn_gates(P, dims, A_log, dt_bias)
        c0 = 2 * dims.Hk * dims.K
        return q_hat, k_hat, P[:, c0:c0 + dims.Hv * dims.V], g, beta

    def gate_exp(self, g):
        return 1.0 - torch.exp(g)

    def log_mul(self, g, factor):
        """g + log(factor): alpha = e^g multiplied by factor."""
        return g + torch.log(factor)

    def mul(self, a, factor):
        return a * factor

    def scan(self, q_hat, k_hat, v, g, beta, B, T, dims, S0=None, form=FORM_PAGES):
        S = torch.empty((B, dims.Hv, dims.K, dims.V), dtype=torch.float32, device=self.dev)
        o, _ = gdn_scan(q_hat, k_hat, v, g, beta, B, T, dims, form=form,
                        algo=SCAN_CHUNKED if T > 1 else SCAN_RECURRENT, state_in=S0, state_out=S)
        return o, S

    def output_gate(self, o, z, w):
        return gdn_output_gate(o, z, w)

    def zeros_like(self, a):
        return torch.zeros_like(a)


# ------------------------------------------------------------------- layer --
@dataclasses.dataclass
class StudyLayer:
    """A GDN layer for the studies: float32 weights (on the backend) and their
    NVFP4 quantisation, gate parameters, dims, output-gate weight."""
    W_in: object
    W_out: object
    W_in_q: object
    W_out_q: object
    A_log: object
    dt_bias: object
    w_norm: object
    dims: GdnDims
    hidden: int

    @staticmethod
    def make(be, W_in, W_out, A_log, dt_bias, dims: GdnDims, hidden: int):
        Wi, Wo = be.upload(W_in), be.upload(W_out)
        return StudyLayer(Wi, Wo, be.quantize(Wi), be.quantize(Wo), be.upload(A_log), be.upload(dt_bias),
                          be.upload(np.ones(dims.V, np.float32)), dims, hidden)

    def slices(self):
        """Column ranges of the fused projection: q|k|v, z, a, b."""
        d = self.dims
        qkv = 2 * d.Hk * d.K + d.Hv * d.V
        z = qkv + d.Hv * d.V
        return {"qkv": (0, qkv), "z": (qkv, z), "a": (z, z + d.Hv), "b": (z + d.Hv, z + 2 * d.Hv)}


def _forward(be, L: StudyLayer, P, B, T, quant_out=False, S0=None):
    """The layer from its fused projection P on: gates, scan, output gate,
    out_proj (W4A4 when quant_out, else unquantised).  Returns (y, S, g, beta)."""
    d = L.dims
    q_hat, k_hat, v, g, beta = be.gates(P, d, L.A_log, L.dt_bias)
    o, S = be.scan(q_hat, k_hat, v, g, beta, B, T, d, S0)
    z0 = L.slices()["z"][0]
    G = be.output_gate(o, P[:, z0:z0 + d.Hv * d.V], L.w_norm)
    G2 = G.reshape(B * T, d.Hv * d.V)
    y = be.w4a4(G2, L.W_out_q) if quant_out else be.matmul_nt(G2, L.W_out)
    return y, S, g, beta, G2


# ------------------------------------------------------ 1. sensitivity replay --
def sensitivity(be, L: StudyLayer, x, B: int, T: int):
    """Per-projection sensitivity replay (Table 3 of the pages).  x: [B*T,
    hidden] activations on the backend.  Returns a dict with one row per
    projection and the joint / root-sum-square comparison."""
    P_c = be.matmul_nt(x, L.W_in)
    P_q = be.w4a4(x, L.W_in_q)
    y_c, S_c, g_c, beta_c, G_c = _forward(be, L, P_c, B, T)
    rows = {}
    for name, (c0, c1) in L.slices().items():
        P = be.copy(P_c)
        be.assign_cols(P, c0, c1, P_q)
        y, S, g, beta, _ = _forward(be, L, P, B, T)
        row = {"gemm_rel": be.rel(P_q[:, c0:c1], P_c[:, c0:c1]), "y_rel": be.rel(y, y_c), "state_rel": be.rel(S, S_c)}
        if name == "a":
            row["one_minus_alpha_rel"] = be.rel(be.gate_exp(g), be.gate_exp(g_c))
        if name == "b":
            row["beta_rel"] = be.rel(beta, beta_c)
        rows[name] = row
    y_o = be.w4a4(G_c, L.W_out_q)
    rows["out"] = {"gemm_rel": be.rel(y_o, y_c), "y_rel": be.rel(y_o, y_c), "state_rel": 0.0}
    y_j, S_j, _, _, _ = _forward(be, L, P_q, B, T, quant_out=True)
    rss = math.sqrt(sum(r["y_rel"] ** 2 for r in rows.values()))
    return {"rows": rows, "joint_y_rel": be.rel(y_j, y_c), "joint_state_rel": be.rel(S_j, S_c), "rss_y_rel": rss}


# ------------------------------------------------------ 2. lockstep / impulse --
def _noise_factors(seed, n_rows, n_cols, sigma):
    g = np.random.Generator(np.random.PCG64(seed))
    return (1.0 + sigma * g.standard_normal((n_rows, n_cols))).astype(np.float32)


def lockstep(be, L: StudyLayer, x, T: int, checkpoints, n_perturbed: int = 11, seed: int = 1234, seg: int = 4096):
    """One clean trajectory and n_perturbed perturbed ones over the same T
    tokens (B = 1 each), carried side by side as the batch of one scan.  The
    first perturbed trajectory uses the W4A4 projections; the others add
    seeded Gaussian noise to each projection at its measured W4A4 error.
    checkpoints: increasing token counts (the last = T).  Returns relS
    (mean and max over the perturbed trajectories) at each checkpoint."""
    d = L.dims
    P_c = be.matmul_nt(x, L.W_in)
    P_q = be.w4a4(x, L.W_in_q)
    sl = L.slices()
    sig = {n: be.rel(P_q[:, a:b], P_c[:, a:b]) for n, (a, b) in sl.items()}
    trajs = [P_c, P_q]
    for j in range(n_perturbed - 1):
        P = be.copy(P_c)
        for i, (n, (a, b)) in enumerate(sl.items()):
            be.scale_cols(P, a, b, be.noise_factors(seed + 100 * j + i, T, b - a, sig[n]))
        trajs.append(P)
    nb = len(trajs)
    # per trajectory: gates once; the scan runs in segments over the batch of trajectories
    per = [be.gates(P, d, L.A_log, L.dt_bias) for P in trajs]
    S = None
    out = []
    t0 = 0
    bounds = []
    for cp in checkpoints:
        while t0 < cp:
            t1 = min(cp, t0 + seg)
            bounds.append((t0, t1, t1 == cp))
            t0 = t1
    for (a, b, at_cp) in bounds:
        cat = [be.cat_rows([p[i][a:b] for p in per]) for i in range(5)]
        _, S = be.scan(*cat, nb, b - a, d, S)
        if at_cp:
            Sh = be.host(S)
            rels = [float(np.linalg.norm(Sh[j] - Sh[0]) / np.linalg.norm(Sh[0])) for j in range(1, nb)]
            out.append({"t": b, "relS_mean": float(np.mean(rels)), "relS_max": float(np.max(rels)),
                        "relS_w4a4": rels[0]})
    return {"projection_sigma": sig, "checkpoints": out}


def impulse(be, L: StudyLayer, x, T: int, t_imp: int = 1024, size: float = 0.01, seed: int = 77,
            phases=((64, 1), (2048, 16)), coarse: int = 256):
    """A state impulse of relative size `size` injected at t_imp into the clean
    trajectory.  The recurrence is affine in the state, so the difference it
    makes evolves as the state of the same scan with v = 0 started from the
    impulse; its norm per value head is read every `step` tokens until `span`
    tokens after the impulse for each (span, step) of `phases`, then every
    `coarse`.  Returns, per head, the steps until the norm falls to 1/e and 1/10
    of the impulse (None when it does not within T) and the horizon
    1/(1 - mean alpha) of that head."""
    d = L.dims
    P_c = be.matmul_nt(x, L.W_in)
    q_hat, k_hat, v, g, beta = be.gates(P_c, d, L.A_log, L.dt_bias)
    _, S1 = be.scan(q_hat[:t_imp], k_hat[:t_imp], v[:t_imp], g[:t_imp], beta[:t_imp], 1, t_imp, d)
    S1h = be.host(S1)
    R = np.random.Generator(np.random.PCG64(seed)).standard_normal(S1h.shape)
    delta = np.empty_like(S1h)
    for h in range(d.Hv):
        delta[0, h] = size * np.linalg.norm(S1h[0, h]) * R[0, h] / np.linalg.norm(R[0, h])
    D = be.upload(delta)
    v0 = be.zeros_like(v)
    n0 = np.linalg.norm(delta[0].reshape(d.Hv, -1), axis=1)
    to_e = [None] * d.Hv
    to_10 = [None] * d.Hv
    t = t_imp
    while t < T and (None in to_e or None in to_10):
        step = next((st for span, st in phases if t - t_imp < span), coarse)
        t1 = min(T, t + step)
        _, D = be.scan(q_hat[t:t1], k_hat[t:t1], v0[t:t1], g[t:t1], beta[t:t1], 1, t1 - t, d, D)
        nd = np.linalg.norm(be.host(D)[0].reshape(d.Hv, -1), axis=1) / n0
        for h in range(d.Hv):
            if to_e[h] is None and nd[h] <= math.exp(-1.0):
                to_e[h] = t1 - t_imp
            if to_10[h] is None and nd[h] <= 0.1:
                to_10[h] = t1 - t_imp
        t = t1
    alpha = np.exp(be.host(g))
    horizon = [float(1.0 / max(1e-12, 1.0 - alpha[:, h].mean())) for h in range(d.Hv)]
    return {"steps_to_1_over_e": to_e, "steps_to_1_over_10": to_10, "horizon_1_over_1_minus_alpha": horizon,
            "resolution": {"phases": [list(p) for p in phases], "after": coarse}}


# -------------------------------------------------------------- 3. gate noise --
def gate_noise(be, L: StudyLayer, x, T: int, alpha_noise: float = 1e-3, beta_noise: float = 1e-2, seed: int = 4321):
    """State error at the end of T tokens after (i) multiplicative noise on
    alpha, (ii) W4A4 on the a projection alone, (iii) multiplicative noise on
    beta (Table 6 of the pages)."""
    d = L.dims
    P_c = be.matmul_nt(x, L.W_in)
    q_hat, k_hat, v, g, beta = be.gates(P_c, d, L.A_log, L.dt_bias)
    _, S_c = be.scan(q_hat, k_hat, v, g, beta, 1, T, d)
    res = {}
    g_n = be.log_mul(g, be.noise_factors(seed, T, d.Hv, alpha_noise))
    _, S = be.scan(q_hat, k_hat, v, g_n, beta, 1, T, d)
    res["alpha_noise"] = {"level": alpha_noise, "state_rel": be.rel(S, S_c)}
    P_q = be.w4a4(x, L.W_in_q)
    a0, a1 = L.slices()["a"]
    P_a = be.copy(P_c)
    be.assign_cols(P_a, a0, a1, P_q)
    _, _, _, g_a, _ = be.gates(P_a, d, L.A_log, L.dt_bias)
    _, S = be.scan(q_hat, k_hat, v, g_a, beta, 1, T, d)
    res["a_quantised"] = {"gemm_rel": be.rel(P_q[:, a0:a1], P_c[:, a0:a1]), "state_rel": be.rel(S, S_c)}
    b_n = be.mul(beta, be.noise_factors(seed + 1, T, d.Hv, beta_noise))
    _, S = be.scan(q_hat, k_hat, v, g, b_n, 1, T, d)
    res["beta_noise"] = {"level": beta_noise, "state_rel": be.rel(S, S_c)}
    return res
