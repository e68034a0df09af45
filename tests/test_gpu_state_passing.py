"""State passing on the GPU (a sequence split into spans joined through the
recurrence's state): the span maps, the state combine and the output
correction against the oracle, then whole segmented scans against the
oracle's recurrence over the unsplit sequence, up to the 32K-token workload
split into eight 4096-token spans."""
import numpy as np
import pytest
import torch

import gdn_synth
import nvfp4_w4a4_gated_b200 as nv
import oracle
from gpu_util import f32_device, rel_fro
from nvfp4_w4a4_gated_b200.seqpar import CudaSpanOps, segmented_scan

pytestmark = pytest.mark.gpu

SCAN_TOL = 2e-3       # the scan's bar (TF32 products inside the chunked kernels)
F32_TOL = 1e-5        # float32 sums of at most 256 products


def _dev_span(arrs, a, e, dims):
    q, k, v, g, beta = (np.ascontiguousarray(x[:, a:e]) for x in arrs)
    B, T = q.shape[0], e - a
    return (f32_device(q.reshape(B * T, dims.Hk, dims.K)), f32_device(k.reshape(B * T, dims.Hk, dims.K)),
            f32_device(v.reshape(B * T, dims.Hv * dims.V)), f32_device(g.reshape(B * T, dims.Hv)),
            f32_device(beta.reshape(B * T, dims.Hv)), T)


@pytest.mark.parametrize("algo", [nv.SCAN_RECURRENT, nv.SCAN_CHUNKED])
@pytest.mark.parametrize("form", [nv.FORM_PAGES, nv.FORM_STANDARD])
@pytest.mark.parametrize("B,T,Hk,Hv,K,V", [
    (1, 1, 1, 2, 128, 128),      # one token
    (2, 64, 2, 4, 128, 64),      # one full chunk; dims.V is not used by the maps
    (1, 130, 2, 2, 64, 128),     # K = 64, ragged last chunk
    (2, 200, 2, 4, 128, 128),
])
def test_transition_matches_oracle(cuda_dev, algo, form, B, T, Hk, Hv, K, V):
    q, k, _, g, beta = gdn_synth.scan_inputs(400 + T, B, T, Hk, Hv, K, V, alpha_lo=0.9, alpha_hi=0.9999)
    dims = nv.GdnDims(Hk, Hv, K, V)
    P, m = nv.gdn_scan_transition(f32_device(q.reshape(B * T, Hk, K)), f32_device(k.reshape(B * T, Hk, K)),
                                  f32_device(g.reshape(B * T, Hv)), f32_device(beta.reshape(B * T, Hv)), B, T, dims,
                                  form=form, algo=algo)
    torch.cuda.synchronize()
    nv.check_device_error()
    P_ref, m_ref = oracle.scan_transition(q, k, g, beta, form=form)
    assert rel_fro(P.cpu().numpy(), P_ref) <= SCAN_TOL
    assert rel_fro(m.cpu().numpy().reshape(B, T, Hv, K), m_ref) <= SCAN_TOL


@pytest.mark.parametrize("K,V", [(32, 32), (64, 128), (128, 128), (128, 64), (64, 256), (128, 96)])
def test_state_combine_matches_oracle(cuda_dev, K, V):
    B, Hv = 2, 3
    P = gdn_synth.gaussian(410, (B, Hv, K, K), std=K ** -0.5)
    S_loc, S_in = gdn_synth.gaussian(411, (B, Hv, K, V)), gdn_synth.gaussian(412, (B, Hv, K, V))
    dP, dL, dI = f32_device(P), f32_device(S_loc), f32_device(S_in)
    out = nv.gdn_state_combine(dP, dL, dI)
    ref = oracle.state_combine(P, S_loc, S_in)
    assert rel_fro(out.cpu().numpy(), ref) <= F32_TOL
    # S_in absent: the local state itself; S_loc absent: the map applied alone
    assert torch.equal(nv.gdn_state_combine(dP, dL, None), dL)
    only = nv.gdn_state_combine(dP, None, dI)
    assert rel_fro(only.cpu().numpy(), oracle.state_combine(P, np.zeros_like(S_loc), S_in)) <= F32_TOL
    # in place on S_in
    nv.gdn_state_combine(dP, dL, dI, out=dI)
    torch.cuda.synchronize()
    assert torch.equal(dI, out)


@pytest.mark.parametrize("K,V", [(64, 64), (128, 128)])
def test_state_combine_chain(cuda_dev, K, V):
    """Five maps composed in one launch equal the oracle's fold, with and
    without a starting state; the result may overwrite the last S_loc."""
    m, B, Hv = 5, 1, 4
    P = gdn_synth.gaussian(415, (m, B, Hv, K, K), std=K ** -0.5)
    S_loc = gdn_synth.gaussian(416, (m, B, Hv, K, V))
    S0 = gdn_synth.gaussian(417, (B, Hv, K, V))
    for start in (None, S0):
        want = None if start is None else start.astype(np.float64)
        for j in range(m):
            want = S_loc[j].astype(np.float64) if want is None else oracle.state_combine(P[j], S_loc[j], want)
        dL = f32_device(S_loc)
        got = nv.gdn_state_combine(f32_device(P), dL, None if start is None else f32_device(start))
        assert rel_fro(got.cpu().numpy(), want) <= F32_TOL
        again = nv.gdn_state_combine(f32_device(P), dL, None if start is None else f32_device(start), out=dL[m - 1])
        torch.cuda.synchronize()
        assert torch.equal(again, got)


@pytest.mark.parametrize("form", [nv.FORM_PAGES, nv.FORM_STANDARD])
@pytest.mark.parametrize("B,T,Hk,Hv,K,V", [
    (2, 200, 2, 4, 128, 128),    # chunked, K == V: one chunk preparation for both
    (1, 64, 1, 2, 64, 64),
    (1, 130, 2, 2, 128, 64),     # K != V: the scan, then the maps
    (2, 1, 1, 2, 128, 128),      # one token
])
def test_scan_span_equals_scan_and_maps(cuda_dev, form, B, T, Hk, Hv, K, V):
    arrs = gdn_synth.scan_inputs(418 + T, B, T, Hk, Hv, K, V, alpha_lo=0.9, alpha_hi=0.9999)
    dims = nv.GdnDims(Hk, Hv, K, V)
    q, k, v, g, beta, _ = _dev_span(arrs, 0, T, dims)
    o, S_loc, P, m = nv.gdn_scan_span(q, k, v, g, beta, B, T, dims, form=form)
    S_ref = torch.empty_like(S_loc)
    o_ref, _ = nv.gdn_scan(q, k, v, g, beta, B, T, dims, form=form, state_out=S_ref)
    P_ref, m_ref = nv.gdn_scan_transition(q, k, g, beta, B, T, dims, form=form)
    torch.cuda.synchronize()
    nv.check_device_error()
    assert torch.equal(o, o_ref) and torch.equal(S_loc, S_ref)
    assert rel_fro(P.cpu().numpy(), P_ref.cpu().numpy()) <= 1e-6
    assert rel_fro(m.cpu().numpy(), m_ref.cpu().numpy()) <= 1e-6
    Po, mo = oracle.scan_transition(arrs[0], arrs[1], arrs[3], arrs[4], form=form)
    assert rel_fro(P.cpu().numpy(), Po) <= SCAN_TOL
    assert rel_fro(m.cpu().numpy().reshape(B, T, Hv, K), mo) <= SCAN_TOL


@pytest.mark.parametrize("variant,tol", [("tcgen05", SCAN_TOL), ("cuda_core", F32_TOL)])
@pytest.mark.parametrize("B,T,Hv,K,V", [
    (1, 1, 2, 128, 128), (2, 100, 4, 128, 128), (1, 64, 3, 64, 128), (2, 65, 2, 128, 64), (1, 130, 2, 64, 64),
    (1, 1000, 5, 128, 128),      # several 128-token tiles per CTA run, heads changing inside a run
])
def test_scan_correct_matches_oracle(cuda_dev, monkeypatch, variant, tol, B, T, Hv, K, V):
    """The tensor-core kernel (TF32 operands, the scan's bar) and the CUDA-core
    kernel (float32) against the oracle; the amax word equals max |o| exactly."""
    if variant == "cuda_core":
        monkeypatch.setenv("NVFP4_CORRECT_VARIANT", "cuda_core")
    o_loc = gdn_synth.gaussian(420, (B, T, Hv, V))
    m = gdn_synth.gaussian(421, (B, T, Hv, K), std=0.1)
    S_in = gdn_synth.gaussian(422, (B, Hv, K, V))
    o = f32_device(o_loc.reshape(B * T, Hv, V))
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.gdn_scan_correct(f32_device(m.reshape(B * T, Hv, K)), f32_device(S_in), o, B, T, amax_word=word)
    torch.cuda.synchronize()
    nv.check_device_error()
    ref = oracle.output_correct(o_loc, m, S_in)
    got = o.cpu().numpy().reshape(B, T, Hv, V)
    assert rel_fro(got, ref) <= tol
    corr = ref - o_loc                 # the correction alone, to its own bar as well
    assert rel_fro(got - o_loc, corr) <= tol
    assert word.view(torch.float32).item() == float(np.abs(got).max())


@pytest.mark.parametrize("form", [nv.FORM_PAGES, nv.FORM_STANDARD])
@pytest.mark.parametrize("bounds", [[0, 64, 100, 200], [0, 1, 130, 200]])
def test_segmented_scan_equals_the_recurrence(cuda_dev, form, bounds):
    B, T, Hk, Hv, K, V = 2, 200, 2, 4, 128, 128
    arrs = gdn_synth.scan_inputs(430, B, T, Hk, Hv, K, V, alpha_lo=0.99, alpha_hi=0.9999)
    S0 = gdn_synth.gaussian(431, (B, Hv, K, V))
    dims = nv.GdnDims(Hk, Hv, K, V)
    spans = [_dev_span(arrs, a, e, dims) for a, e in zip(bounds, bounds[1:])]
    outs, S = segmented_scan(spans, B, dims, form=form, state_in=f32_device(S0))
    torch.cuda.synchronize()
    nv.check_device_error()
    o_ref, S_ref = oracle.scan(*arrs, form=form, S0=S0)
    got = np.concatenate([o.cpu().numpy().reshape(B, -1, Hv, V) for o in outs], axis=1)
    assert rel_fro(got, o_ref) <= SCAN_TOL
    assert rel_fro(S.cpu().numpy(), S_ref) <= SCAN_TOL
    # the joins matter: the last span's zero-start outputs are far from the truth
    o_last, _ = oracle.scan(*(x[:, bounds[-2]:] for x in arrs), form=form)
    assert rel_fro(o_last, o_ref[:, bounds[-2]:]) > 0.1


def test_segmented_scan_32k_in_eight_spans(cuda_dev):
    """T = 32768, 16 key / 32 value heads of 128 (the long-context workload),
    split into eight spans of 4096 tokens: against the unsplit GPU scan on all
    heads, and against the oracle's recurrence on value heads 5 and 30."""
    B, T, Hk, Hv, K, V = 1, 32768, 16, 32, 128, 128
    arrs = gdn_synth.scan_inputs(440, B, T, Hk, Hv, K, V, alpha_lo=0.99, alpha_hi=0.9999)
    dims = nv.GdnDims(Hk, Hv, K, V)
    whole = _dev_span(arrs, 0, T, dims)
    S_whole = torch.empty((B, Hv, K, V), device="cuda")
    o_whole, _ = nv.gdn_scan(*whole[:5], B, T, dims, state_out=S_whole)
    bounds = list(range(0, T + 1, 4096))
    spans = [tuple(x[a:e] for x in whole[:5]) + (e - a,) for a, e in zip(bounds, bounds[1:])]
    outs, S = segmented_scan(spans, B, dims)
    torch.cuda.synchronize()
    nv.check_device_error()
    o_seg = torch.cat(outs)
    assert rel_fro(o_seg.cpu().numpy(), o_whole.cpu().numpy()) <= SCAN_TOL
    assert rel_fro(S.cpu().numpy(), S_whole.cpu().numpy()) <= SCAN_TOL
    o_seg = o_seg.cpu().numpy().reshape(B, T, Hv, V)
    S = S.cpu().numpy()
    q, k, v, g, beta = arrs
    for h in (5, 30):
        hk = h * Hk // Hv
        o_ref, S_ref = oracle.scan(q[:, :, hk:hk + 1], k[:, :, hk:hk + 1], v[:, :, h:h + 1], g[:, :, h:h + 1],
                                   beta[:, :, h:h + 1])
        assert rel_fro(o_seg[:, :, h:h + 1], o_ref) <= SCAN_TOL
        assert rel_fro(S[:, h:h + 1], S_ref) <= SCAN_TOL
