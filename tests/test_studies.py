"""The mechanism studies (review page, paper sec.5.2 Table 3 and sec.5.3 Fig. 1,
Table 6) run with the oracle's steps on the tiny layer: the study code is
checked against what it must reproduce by construction.  Their numbers on
random weights are context, not a reproduction of the pages' (parity
unpinned: the pages measure a trained model)."""
import math

import numpy as np
import pytest

import gdn_synth
import oracle
from nvfp4_w4a4_gated_b200 import GdnDims
from nvfp4_w4a4_gated_b200 import studies
from study_oracle_backend import OracleBackend


def _tiny(seed=40, T=64, B=1):
    sh = gdn_synth.TINY
    be = OracleBackend()
    dims = GdnDims(sh.Hk, sh.Hv, sh.K, sh.V)
    W_in = gdn_synth.weights(seed, sh.n_in, sh.H)
    W_out = gdn_synth.weights(seed + 1, sh.H, sh.Hv * sh.V)
    A_log, dt_bias = gdn_synth.gate_params(seed + 2, sh.Hv)
    _, x = gdn_synth.activations(seed + 3, B * T, sh.H, hot="fixed")
    L = studies.StudyLayer.make(be, W_in, W_out, A_log, dt_bias, dims, sh.H)
    return be, L, x, (W_in, W_out, A_log, dt_bias), sh


def test_sensitivity_joint_row_is_the_w4a4_layer():
    """The joint row quantises every projection: its y is the oracle's W4A4
    layer with the output gate (unit weight), and its error is measured against
    the same layer with no quantisation at all, both formed here straight from
    the oracle's functions."""
    be, L, x, (W_in, W_out, A_log, dt_bias), sh = _tiny()
    r = studies.sensitivity(be, L, x, 1, 64)
    y_q = oracle.layer_forward(x, oracle.quantize(W_in), oracle.quantize(W_out), A_log, dt_bias, 1, 64, sh.Hk, sh.Hv,
                               sh.K, sh.V, out_norm=np.ones(sh.V))[0]
    P = oracle.gemm_nt(x, W_in)
    q, k, v, z, a, b = oracle.split_projection(P, sh.Hk, sh.Hv, sh.K, sh.V)
    g, beta = oracle.gates(a, b, A_log, dt_bias)
    o, _ = oracle.scan(oracle.l2norm(q.reshape(1, 64, sh.Hk, sh.K)), oracle.l2norm(k.reshape(1, 64, sh.Hk, sh.K)),
                       v.reshape(1, 64, sh.Hv, sh.V), g.reshape(1, 64, sh.Hv), beta.reshape(1, 64, sh.Hv))
    G = oracle.output_gate(o.reshape(64, sh.Hv, sh.V).astype(np.float32), z.reshape(64, sh.Hv, sh.V), np.ones(sh.V))
    y_c = oracle.gemm_nt(G.reshape(64, -1), W_out)
    assert abs(r["joint_y_rel"] - np.linalg.norm(y_q - y_c) / np.linalg.norm(y_c)) < 1e-12
    rows = r["rows"]
    assert set(rows) == {"qkv", "z", "a", "b", "out"}
    c1 = 2 * sh.Hk * sh.K + sh.Hv * sh.V
    P_q = oracle.w4a4_gemm(oracle.quantize(x), oracle.quantize(W_in))
    assert abs(rows["qkv"]["gemm_rel"] - np.linalg.norm(P_q[:, :c1] - P[:, :c1]) / np.linalg.norm(P[:, :c1])) < 1e-12
    for name in ("qkv", "z", "a", "b", "out"):
        assert 0.0 < rows[name]["gemm_rel"] < 0.5 and 0.0 < rows[name]["y_rel"] < 1.0
    assert abs(r["rss_y_rel"] - math.sqrt(sum(row["y_rel"] ** 2 for row in rows.values()))) < 1e-15
    assert rows["a"]["one_minus_alpha_rel"] > 0 and rows["b"]["beta_rel"] > 0


def test_sensitivity_nothing_quantised_moves_nothing():
    """With the W4A4 products replaced by the unquantised ones, every error is 0."""
    be, L, x, _, _ = _tiny()

    class Exact(OracleBackend):
        def w4a4(self, x, Wq):
            return super().matmul_nt(x, self._W[id(Wq)])

    ex = Exact()
    ex._W = {id(L.W_in_q): L.W_in, id(L.W_out_q): L.W_out}
    r = studies.sensitivity(ex, L, x, 1, 64)
    assert all(v == 0.0 for row in r["rows"].values() for v in row.values())
    assert r["joint_y_rel"] == 0.0 and r["rss_y_rel"] == 0.0


def test_lockstep_clean_and_w4a4_trajectories():
    """relS is 0 for identical trajectories and positive for perturbed ones;
    the W4A4 trajectory's final state is the oracle scan of the W4A4
    projections (the lockstep batch carries each trajectory independently)."""
    be, L, x, (W_in, _, A_log, dt_bias), sh = _tiny(T=96)
    res = studies.lockstep(be, L, x, 96, [32, 64, 96], n_perturbed=3, seg=40)
    cps = res["checkpoints"]
    assert [c["t"] for c in cps] == [32, 64, 96]
    assert all(c["relS_mean"] > 0 and c["relS_max"] >= c["relS_mean"] for c in cps)
    # the W4A4 trajectory alone, through the oracle, from scratch
    P_q = oracle.w4a4_gemm(oracle.quantize(x), oracle.quantize(W_in))
    P_c = oracle.gemm_nt(x, W_in)
    d = L.dims
    def final_state(P):
        q, k, v, g, b = be.gates(P, d, A_log, dt_bias)
        return be.scan(q, k, v, g, b, 1, 96, d)[1]
    S_q, S_c = final_state(P_q), final_state(P_c)
    want = np.linalg.norm(S_q - S_c) / np.linalg.norm(S_c)
    assert abs(cps[-1]["relS_w4a4"] - want) < 1e-9


def test_impulse_is_the_state_difference():
    """The impulse response read from the v = 0 scan equals the difference of
    two full recurrences (with and without the impulse): the recurrence is
    affine in the state.  Its norm never grows (every token's map has spectral
    norm <= 1 for unit keys, alpha, beta in (0, 1))."""
    be, L, x, (W_in, _, A_log, dt_bias), sh = _tiny(T=256)
    res = studies.impulse(be, L, x, 256, t_imp=64, phases=((16, 1), (64, 8)), coarse=32)
    assert len(res["steps_to_1_over_e"]) == L.dims.Hv
    for e, t10 in zip(res["steps_to_1_over_e"], res["steps_to_1_over_10"]):
        assert e is None or t10 is None or e <= t10
    # independent check at t = 64 + 40: full recurrence with and without the impulse
    d = L.dims
    P = oracle.gemm_nt(x, W_in)
    q, k, v, g, b = be.gates(P, d, A_log, dt_bias)
    _, S1 = be.scan(q[:64], k[:64], v[:64], g[:64], b[:64], 1, 64, d)
    rng = np.random.Generator(np.random.PCG64(77)).standard_normal(S1.shape)
    delta = np.stack([0.01 * np.linalg.norm(S1[0, h]) * rng[0, h] / np.linalg.norm(rng[0, h]) for h in range(d.Hv)])[None]
    _, Sa = be.scan(q[64:104], k[64:104], v[64:104], g[64:104], b[64:104], 1, 40, d, S1 + delta)
    _, Sb = be.scan(q[64:104], k[64:104], v[64:104], g[64:104], b[64:104], 1, 40, d, S1)
    _, D = be.scan(q[64:104], k[64:104], np.zeros_like(v[64:104]), g[64:104], b[64:104], 1, 40, d, delta)
    assert np.allclose(Sa - Sb, D, rtol=1e-9, atol=1e-12 * np.abs(delta).max())
    norms = []
    Dt = delta
    for t in range(64, 104):
        _, Dt = be.scan(q[t:t + 1], k[t:t + 1], np.zeros_like(v[t:t + 1]), g[t:t + 1], b[t:t + 1], 1, 1, d, Dt)
        norms.append(np.linalg.norm(Dt))
    assert all(n1 <= n0 * (1 + 1e-12) for n0, n1 in zip([np.linalg.norm(delta)] + norms, norms))


def test_gate_noise_levels_and_zero_noise():
    """Zero noise leaves the state unchanged; the table's rows carry the levels asked for."""
    be, L, x, _, _ = _tiny()
    res = studies.gate_noise(be, L, x, 64, alpha_noise=0.0, beta_noise=0.0)
    assert res["alpha_noise"]["state_rel"] == 0.0 and res["beta_noise"]["state_rel"] == 0.0
    assert res["a_quantised"]["gemm_rel"] > 0 and res["a_quantised"]["state_rel"] > 0
    res = studies.gate_noise(be, L, x, 64)
    assert res["alpha_noise"]["level"] == 1e-3 and res["beta_noise"]["level"] == 1e-2
    assert res["alpha_noise"]["state_rel"] > 0 and res["beta_noise"]["state_rel"] > 0
