"""Gates, q/k normalisation and the delta-rule scan on the GPU vs the oracle
(float64).  Gates: relative 1e-5 elementwise; scan outputs and final state:
relative Frobenius error <= 2e-3."""
import math

import numpy as np
import pytest
import torch

import gdn_synth
import nvfp4_w4a4_gated_b200 as nv
import oracle
from gpu_util import f32_device, rel_fro

pytestmark = pytest.mark.gpu

SCAN_TOL = 2e-3


@pytest.mark.parametrize("n,Hk,Hv,K,V", [(64, 2, 2, 64, 64), (300, 16, 32, 128, 128), (5, 1, 4, 128, 64)])
def test_gates_match_oracle(cuda_dev, n, Hk, Hv, K, V):
    dims = nv.GdnDims(Hk, Hv, K, V)
    g0 = gdn_synth.rng(n + Hv)
    P = (g0.standard_normal((n, dims.n_in)) * 3).astype(np.float32)
    A_log, dt_bias = gdn_synth.gate_params(7, Hv)
    q_hat, k_hat, g, beta = nv.gdn_gates(f32_device(P), dims, f32_device(A_log), f32_device(dt_bias))
    torch.cuda.synchronize()
    q, k, _v, _z, a, b = oracle.split_projection(P.astype(np.float64), Hk, Hv, K, V)
    g_ref, b_ref = oracle.gates(a, b, A_log, dt_bias)
    assert np.allclose(g.cpu().numpy(), g_ref, rtol=1e-5, atol=0)
    assert np.allclose(beta.cpu().numpy(), b_ref, rtol=1e-5, atol=0)
    assert np.allclose(q_hat.cpu().numpy(), oracle.l2norm(q.reshape(n, Hk, K)), rtol=0, atol=1e-6)
    assert np.allclose(k_hat.cpu().numpy(), oracle.l2norm(k.reshape(n, Hk, K)), rtol=0, atol=1e-6)


def _scan_case(B, T, Hk, Hv, K, V, seed, form, algo, state=True, alpha=(0.9, 0.9999)):
    q, k, v, g, beta = gdn_synth.scan_inputs(seed, B, T, Hk, Hv, K, V, alpha_lo=alpha[0], alpha_hi=alpha[1])
    S0 = gdn_synth.gaussian(seed + 1, (B, Hv, K, V), std=0.3) if state else None
    dims = nv.GdnDims(Hk, Hv, K, V)
    s_out = torch.empty((B, Hv, K, V), dtype=torch.float32, device="cuda")
    o, _ = nv.gdn_scan(f32_device(q.reshape(B * T, Hk, K)), f32_device(k.reshape(B * T, Hk, K)),
                       f32_device(v.reshape(B * T, Hv * V)), f32_device(g.reshape(B * T, Hv)),
                       f32_device(beta.reshape(B * T, Hv)), B, T, dims, form=form, algo=algo,
                       state_in=None if S0 is None else f32_device(S0), state_out=s_out)
    torch.cuda.synchronize()
    nv.check_device_error()
    o_ref, S_ref = oracle.scan(q, k, v, g, beta, form=form, S0=S0)
    return o.cpu().numpy().reshape(B, T, Hv, V), s_out.cpu().numpy(), o_ref, S_ref


@pytest.mark.parametrize("algo", [nv.SCAN_RECURRENT, nv.SCAN_CHUNKED])
@pytest.mark.parametrize("form", [nv.FORM_PAGES, nv.FORM_STANDARD])
@pytest.mark.parametrize("B,T,Hk,Hv,K,V", [
    (1, 64, 1, 2, 64, 64),       # one full chunk
    (2, 200, 2, 4, 128, 128),    # ragged last chunk, GQA 2 value heads per key head
    (1, 1, 1, 2, 128, 64),       # one token (decode)
    (1, 130, 2, 2, 64, 128),     # K != V
])
def test_scan_matches_oracle(cuda_dev, algo, form, B, T, Hk, Hv, K, V):
    o, S, o_ref, S_ref = _scan_case(B, T, Hk, Hv, K, V, 11 + T, form, algo)
    assert rel_fro(o, o_ref) <= SCAN_TOL
    assert rel_fro(S, S_ref) <= SCAN_TOL


@pytest.mark.parametrize("algo", [nv.SCAN_RECURRENT, nv.SCAN_CHUNKED])
def test_scan_long_memory(cuda_dev, algo):
    """alpha in (0.99, 0.9999): the state carries over all 16 chunks."""
    o, S, o_ref, S_ref = _scan_case(1, 1000, 1, 2, 128, 128, 5, nv.FORM_PAGES, algo, alpha=(0.99, 0.9999))
    assert rel_fro(o, o_ref) <= SCAN_TOL
    assert rel_fro(S, S_ref) <= SCAN_TOL


@pytest.mark.parametrize("t,tol", [(128, 1e-6), (100, SCAN_TOL)])
def test_scan_chaining_on_gpu(cuda_dev, t, tol):
    """scan(0..T) equals scan(0..t) then scan(t..T) from the carried state: to
    float32 rounding when t is a chunk boundary, to the scan bar otherwise
    (the chunk boundaries, hence the TF32 rounding, move)."""
    B, T, Hk, Hv, K, V = 1, 300, 1, 2, 128, 128
    q, k, v, g, beta = gdn_synth.scan_inputs(21, B, T, Hk, Hv, K, V)
    dims = nv.GdnDims(Hk, Hv, K, V)
    dev = lambda a: f32_device(a)
    full_s = torch.empty((B, Hv, K, V), device="cuda")
    o_full, _ = nv.gdn_scan(dev(q[0]), dev(k[0]), dev(v[0].reshape(T, -1)), dev(g[0]), dev(beta[0]), B, T, dims,
                            state_out=full_s)
    mid = torch.empty_like(full_s)
    o1, _ = nv.gdn_scan(dev(q[0, :t]), dev(k[0, :t]), dev(v[0, :t].reshape(t, -1)), dev(g[0, :t]), dev(beta[0, :t]),
                        B, t, dims, state_out=mid)
    end = torch.empty_like(full_s)
    o2, _ = nv.gdn_scan(dev(q[0, t:]), dev(k[0, t:]), dev(v[0, t:].reshape(T - t, -1)), dev(g[0, t:]),
                        dev(beta[0, t:]), B, T - t, dims, state_in=mid, state_out=end)
    torch.cuda.synchronize()
    assert rel_fro(torch.cat([o1, o2]).cpu().numpy(), o_full.cpu().numpy()) <= tol
    assert rel_fro(end.cpu().numpy(), full_s.cpu().numpy()) <= tol


def test_scan_full_size_subset_of_heads(cuda_dev):
    """T = 4096, 16 key / 32 value heads, K = V = 128 (the layer-prefill scan
    launch); the oracle recomputes value heads 0, 1 and 31."""
    B, T, Hk, Hv, K, V = 1, 4096, 16, 32, 128, 128
    q, k, v, g, beta = gdn_synth.scan_inputs(33, B, T, Hk, Hv, K, V, alpha_lo=0.5, alpha_hi=0.999)
    dims = nv.GdnDims(Hk, Hv, K, V)
    s_out = torch.empty((B, Hv, K, V), dtype=torch.float32, device="cuda")
    o, _ = nv.gdn_scan(f32_device(q[0]), f32_device(k[0]), f32_device(v[0].reshape(T, -1)), f32_device(g[0]),
                       f32_device(beta[0]), B, T, dims, state_out=s_out)
    torch.cuda.synchronize()
    o = o.cpu().numpy().reshape(B, T, Hv, V)
    s = s_out.cpu().numpy()
    for h in (0, 1, 31):
        hk = h * Hk // Hv
        o_ref, S_ref = oracle.scan(q[:, :, hk:hk + 1], k[:, :, hk:hk + 1], v[:, :, h:h + 1], g[:, :, h:h + 1],
                                   beta[:, :, h:h + 1])
        assert rel_fro(o[:, :, h:h + 1], o_ref) <= SCAN_TOL
        assert rel_fro(s[:, h:h + 1], S_ref) <= SCAN_TOL


def test_scan_state_impulse_decay(cuda_dev):
    """A 1% state impulse injected at t = 1000 (as in the long-context workload)
    evolves as D_t = (alpha_t I - beta_t k k^T) D_{t-1}, independently of v
    (review page, mechanism step 3, impulse study): the GPU scan started from
    D with v = 0 must follow the oracle's direct product at checkpoints."""
    B, T, Hk, Hv, K, V, t_imp = 1, 1000 + 512, 1, 1, 128, 128, 1000
    q, k, v, g, beta = gdn_synth.scan_inputs(41, B, T, Hk, Hv, K, V, alpha_lo=0.95, alpha_hi=0.9999)
    dims = nv.GdnDims(Hk, Hv, K, V)
    _, S_mid = oracle.scan(q[:, :t_imp], k[:, :t_imp], v[:, :t_imp], g[:, :t_imp], beta[:, :t_imp])
    R = gdn_synth.gaussian(42, S_mid.shape).astype(np.float64)
    D0 = 0.01 * np.linalg.norm(S_mid) * R / np.linalg.norm(R)
    zeros_v = np.zeros((T - t_imp, Hv * V), np.float32)
    for span in (1, 2, 8, 64, 256, 512):
        sl = slice(t_imp, t_imp + span)
        s = torch.empty((B, Hv, K, V), device="cuda")
        nv.gdn_scan(f32_device(q[0, sl]), f32_device(k[0, sl]), f32_device(zeros_v[:span]), f32_device(g[0, sl]),
                    f32_device(beta[0, sl]), B, span, dims, state_in=f32_device(D0), state_out=s)
        torch.cuda.synchronize()
        D = D0[0, 0].copy()
        for t in range(t_imp, t_imp + span):
            kt = k[0, t, 0].astype(np.float64)
            D = math.exp(g[0, t, 0]) * D - beta[0, t, 0] * np.outer(kt, kt @ D)
        assert rel_fro(s.cpu().numpy()[0, 0], D) <= SCAN_TOL
        assert np.linalg.norm(D) < np.linalg.norm(D0) * 1.0001
