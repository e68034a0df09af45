"""gdn_layer_forward on the GPU vs the oracle's layer, stage by stage.

Stages whose inputs are identical on both sides are held to the kernel bars
(bit-exact quantisation, 1e-3 GEMM, 2e-3 scan).  Downstream of the scan the
two sides quantise slightly different o (TF32 vs float64), so a few codes on
rounding boundaries differ; there the check is the fraction of differing
codes and the layer output at the W4A4 noise level."""
import numpy as np
import pytest
import torch

import gdn_synth
import nvfp4_w4a4_gated_b200 as nv
import oracle
from gpu_util import bf16_device, f32_device, rel_fro

pytestmark = pytest.mark.gpu


def _view(ws, off, nbytes, dtype):
    return ws[off:off + nbytes].view(dtype)


def _make_layer(shape, seed, dev="cuda"):
    W_in = gdn_synth.weights(seed + 100, shape.n_in, shape.H)
    W_out = gdn_synth.weights(seed + 101, shape.H, shape.Hv * shape.V)
    A_log, dt_bias = gdn_synth.gate_params(seed + 102, shape.Hv)
    dims = nv.GdnDims(shape.Hk, shape.Hv, shape.K, shape.V)
    w = nv.LayerWeights(nv.nvfp4_quantize(f32_device(W_in)), nv.nvfp4_quantize(f32_device(W_out)),
                        f32_device(A_log), f32_device(dt_bias), dims, shape.H)
    return w, (W_in, W_out, A_log, dt_bias)


@pytest.mark.parametrize("form", [nv.FORM_PAGES, nv.FORM_STANDARD])
@pytest.mark.parametrize("B,T", [(1, 64), (2, 100)])   # (2, 100): two sequences, a ragged last chunk
def test_tiny_layer_stagewise(cuda_dev, form, B, T):
    sh = gdn_synth.TINY
    bits, x = gdn_synth.activations(0, B * T, sh.H, hot="fixed")
    w, (W_in, W_out, A_log, dt_bias) = _make_layer(sh, 0)
    S_out = torch.empty((B, sh.Hv, sh.K, sh.V), device="cuda")
    y, ws, lay = nv.gdn_layer_forward(w, bf16_device(bits), B, T, state_out=S_out, form=form)
    torch.cuda.synchronize()
    nv.check_device_error()
    ref = oracle.layer_forward(x, oracle.quantize(W_in), oracle.quantize(W_out), A_log, dt_bias, B, T, sh.Hk, sh.Hv,
                               sh.K, sh.V, form=form, stages=True)
    BT, H, n_in, HvV = B * T, sh.H, sh.n_in, sh.Hv * sh.V
    ldp = (n_in + 3) // 4 * 4
    # stage 1: activation quantisation, bit-exact
    xc = _view(ws, lay["x_codes"], BT * H // 2, torch.uint8).cpu().numpy().reshape(BT, H // 2)
    assert np.array_equal(xc, ref["xq"][0])
    xsf = ws[lay["x_sf"]:lay["x_sf"] + nv.lib().nvfp4_sf_bytes(BT, H)].cpu().numpy()
    assert np.array_equal(xsf, oracle.sf_linear_to_mma(ref["xq"][1], BT, H))
    # stage 2: fused in_proj GEMM (same quantised operands on both sides)
    P = _view(ws, lay["proj"], BT * ldp * 4, torch.float32).cpu().numpy().reshape(BT, ldp)[:, :n_in]
    assert rel_fro(P, ref["P"]) <= 1e-3
    # stage 3: gates and normalisation
    g = _view(ws, lay["g"], BT * sh.Hv * 4, torch.float32).cpu().numpy().reshape(BT, sh.Hv)
    beta = _view(ws, lay["beta"], BT * sh.Hv * 4, torch.float32).cpu().numpy().reshape(BT, sh.Hv)
    assert rel_fro(g, ref["g"]) <= 1e-3 and rel_fro(beta, ref["beta"]) <= 1e-3
    # stage 4: the scan and the state
    o = _view(ws, lay["o"], BT * HvV * 4, torch.float32).cpu().numpy().reshape(B, T, sh.Hv, sh.V)
    assert rel_fro(o, ref["o"]) <= 2e-3
    assert rel_fro(S_out.cpu().numpy(), ref["S"]) <= 2e-3
    # stage 5: o quantisation: nearly all codes agree (inputs differ at the 1e-4 level)
    oc = _view(ws, lay["o_codes"], BT * HvV // 2, torch.uint8).cpu().numpy().reshape(BT, HvV // 2)
    flipped = np.mean(oc != ref["oq"][0])
    assert flipped < 0.02
    # stage 6: layer output.  A flipped code moves its element by one E2M1 step, at most
    # half its magnitude, so the output moves by about 0.5 sqrt(flipped) relative; the
    # out_proj itself is held to 1e-3 in the isolated test below.
    assert rel_fro(y.cpu().numpy(), ref["y"]) <= max(2e-2, 0.5 * np.sqrt(flipped))


def test_tiny_layer_out_proj_stage_isolated(cuda_dev):
    """The out_proj stage fed the oracle's own quantised o: 1e-3 GEMM bar."""
    sh, B, T = gdn_synth.TINY, 1, 64
    _, x = gdn_synth.activations(0, B * T, sh.H, hot="fixed")
    W_in = gdn_synth.weights(100, sh.n_in, sh.H)
    W_out = gdn_synth.weights(101, sh.H, sh.Hv * sh.V)
    A_log, dt_bias = gdn_synth.gate_params(102, sh.Hv)
    ref = oracle.layer_forward(x, oracle.quantize(W_in), oracle.quantize(W_out), A_log, dt_bias, B, T, sh.Hk, sh.Hv,
                               sh.K, sh.V, stages=True)
    from gpu_util import upload_oracle_nvfp4
    oq = upload_oracle_nvfp4(ref["oq"], B * T, sh.Hv * sh.V)
    wq = upload_oracle_nvfp4(oracle.quantize(W_out), sh.H, sh.Hv * sh.V)
    y = nv.w4a4_gemm(oq, wq)
    torch.cuda.synchronize()
    assert rel_fro(y.cpu().numpy(), ref["y"]) <= 1e-3


def test_layer_decode_step_chain(cuda_dev):
    """Decode: T = 1 per call, B = 3 sequences, the state carried in place over four
    steps.  Each step is checked against the oracle's layer step taken from the
    oracle's own carried state: o and the state within the scan bar, the o codes and
    y at the flip bar of the stage-wise test (each single-token call quantises its
    own rows with its own per-tensor scale, on both sides)."""
    sh, B, steps = gdn_synth.TINY, 3, 4
    w, (W_in, W_out, A_log, dt_bias) = _make_layer(sh, 7)
    bits, x = gdn_synth.activations(8, B * steps, sh.H, hot="fixed")
    xs = bf16_device(bits).view(B, steps, sh.H)
    xh = x.reshape(B, steps, sh.H)
    Wq_in, Wq_out = oracle.quantize(W_in), oracle.quantize(W_out)
    W_in_deq, W_out_deq = oracle.dequantize(*Wq_in), oracle.dequantize(*Wq_out)
    S = torch.zeros((B, sh.Hv, sh.K, sh.V), device="cuda")
    S_ref = np.zeros((B, sh.Hv, sh.K, sh.V))
    HvV = sh.Hv * sh.V
    for t in range(steps):
        y, ws, lay = nv.gdn_layer_forward(w, xs[:, t].contiguous(), B, 1, state_in=S, state_out=S)
        torch.cuda.synchronize()
        nv.check_device_error()
        ref = oracle.layer_forward(np.ascontiguousarray(xh[:, t]), Wq_in, Wq_out, A_log, dt_bias, B, 1, sh.Hk, sh.Hv,
                                   sh.K, sh.V, S0=S_ref, stages=True, W_in_deq=W_in_deq, W_out_deq=W_out_deq)
        o = _view(ws, lay["o"], B * HvV * 4, torch.float32).cpu().numpy().reshape(B, 1, sh.Hv, sh.V)
        assert rel_fro(o, ref["o"]) <= 2e-3, t
        assert rel_fro(S.cpu().numpy(), ref["S"]) <= 2e-3, t
        oc = _view(ws, lay["o_codes"], B * HvV // 2, torch.uint8).cpu().numpy().reshape(B, HvV // 2)
        flipped = np.mean(oc != ref["oq"][0])
        assert flipped < 0.02, t
        assert rel_fro(y.cpu().numpy(), ref["y"]) <= max(2e-2, 0.5 * np.sqrt(flipped)), t
        S_ref = ref["S"]
    assert np.linalg.norm(S_ref) > 0


def test_full_size_prefill_layer_stage_checks(cuda_dev):
    """The T = 4096 layer-prefill workload (hidden 5120, 16/32 heads, K = V = 128)
    in the launch configuration the benchmark times: bit-exact activation
    quantisation, sampled rows of the fused projection against the float64
    oracle, finite outputs."""
    sh, B, T = gdn_synth.FULL, 1, 4096
    bits, x = gdn_synth.activations(2, B * T, sh.H, hot="percent")
    w, (W_in, W_out, A_log, dt_bias) = _make_layer(sh, 2)
    S_out = torch.empty((B, sh.Hv, sh.K, sh.V), device="cuda")
    y, ws, lay = nv.gdn_layer_forward(w, bf16_device(bits), B, T, state_out=S_out)
    torch.cuda.synchronize()
    nv.check_device_error()
    BT, H, n_in = B * T, sh.H, sh.n_in
    xq = oracle.quantize(x)
    xc = _view(ws, lay["x_codes"], BT * H // 2, torch.uint8).cpu().numpy().reshape(BT, H // 2)
    assert np.array_equal(xc, xq[0])
    Wq = oracle.quantize(W_in)
    rows = np.array([0, 1, 777, 2048, 4095])
    Ad = oracle.dequantize(xq[0][rows], xq[1][rows], xq[2])
    ref = oracle.gemm_nt(Ad, oracle.dequantize(*Wq))
    ldp = (n_in + 3) // 4 * 4
    P = _view(ws, lay["proj"], BT * ldp * 4, torch.float32).view(BT, ldp)[torch.from_numpy(rows).cuda(), :n_in]
    assert rel_fro(P.cpu().numpy(), ref) <= 1e-3
    assert torch.isfinite(y).all() and torch.isfinite(S_out).all()


def test_prefill_T32768_projections_sampled_rows(cuda_dev):
    """The T = 32768 layer prefill as the benchmark runs it (one call).  Both GEMMs
    have M > N there, so the n tiles of one m tile run back to back.  On sampled
    rows: x codes bit-exact; P against the float64 product of the oracle-quantised
    operands; y against the oracle's product of the GPU's o, quantised under the
    GPU's o scale, with W_out (the o codes themselves are checked bit for bit by
    the o-quantiser tests)."""
    sh, B, T = gdn_synth.FULL, 1, 32768
    bits, x = gdn_synth.activations(3, B * T, sh.H, hot="percent")
    w, (W_in, W_out, _, _) = _make_layer(sh, 3)
    y, ws, lay = nv.gdn_layer_forward(w, bf16_device(bits), B, T)
    torch.cuda.synchronize()
    nv.check_device_error()
    BT, H, n_in, HvV = B * T, sh.H, sh.n_in, sh.Hv * sh.V
    ldp = (n_in + 3) // 4 * 4
    rows = np.unique(np.concatenate([np.arange(4), gdn_synth.rng(9).integers(0, BT, 24), np.arange(BT - 4, BT)]))
    rows_t = torch.from_numpy(rows).cuda()
    xq = oracle.quantize(x)
    xc = _view(ws, lay["x_codes"], BT * H // 2, torch.uint8).view(BT, H // 2)[rows_t].cpu().numpy()
    assert np.array_equal(xc, xq[0][rows])
    ref_P = oracle.gemm_nt(oracle.dequantize(xq[0][rows], xq[1][rows], xq[2]), oracle.dequantize(*oracle.quantize(W_in)))
    P = _view(ws, lay["proj"], BT * ldp * 4, torch.float32).view(BT, ldp)[rows_t, :n_in].cpu().numpy()
    assert rel_fro(P, ref_P) <= 1e-3
    o = _view(ws, lay["o"], BT * HvV * 4, torch.float32).view(BT, HvV)[rows_t].cpu().numpy()
    oS = float(_view(ws, lay["o_scale"], 4, torch.float32).cpu().numpy()[0])
    ref_y = oracle.gemm_nt(oracle.dequantize(*oracle.quantize(o, S=oS)), oracle.dequantize(*oracle.quantize(W_out)))
    got_y = y[rows_t].cpu().numpy()
    assert rel_fro(got_y, ref_y) <= 1e-3
    assert np.max(np.abs(got_y - ref_y)) <= 1e-3 * np.max(np.abs(ref_y))


def _check_o_quantised_exactly(ws, lay, BT, HvV, o_field="o"):
    """The o quantiser in the layer takes its amax from the word the scan (or the
    output gate) filled, and runs only its quantisation pass.  Codes, block scales
    and the global scale must equal the oracle's quantisation of the same o."""
    o = _view(ws, lay[o_field], BT * HvV * 4, torch.float32).cpu().numpy().reshape(BT, HvV)
    codes, sf, S = oracle.quantize(o)
    oc = _view(ws, lay["o_codes"], BT * HvV // 2, torch.uint8).cpu().numpy().reshape(BT, HvV // 2)
    osf = ws[lay["o_sf"]:lay["o_sf"] + nv.lib().nvfp4_sf_bytes(BT, HvV)].cpu().numpy()
    oS = _view(ws, lay["o_scale"], 4, torch.float32).cpu().numpy()[0]
    assert np.float32(oS) == np.float32(S)
    assert np.array_equal(oc, codes)
    assert np.array_equal(osf, oracle.sf_linear_to_mma(sf, BT, HvV))


@pytest.mark.parametrize("B,T", [(1, 64), (2, 100), (3, 1)])   # chunked scan twice, then the one-token scan
def test_o_quantised_from_the_producer_amax(cuda_dev, B, T):
    sh = gdn_synth.TINY
    bits, _ = gdn_synth.activations(5, B * T, sh.H, hot="fixed")
    w, _ = _make_layer(sh, 5)
    S0 = f32_device(gdn_synth.gaussian(6, (B, sh.Hv, sh.K, sh.V), std=0.5))
    _, ws, lay = nv.gdn_layer_forward(w, bf16_device(bits), B, T, state_in=S0)
    torch.cuda.synchronize()
    nv.check_device_error()
    _check_o_quantised_exactly(ws, lay, B * T, sh.Hv * sh.V)


def test_o_quantised_from_the_producer_amax_full_size(cuda_dev):
    """The T = 4096 layer-prefill workload as the benchmark runs it."""
    sh, B, T = gdn_synth.FULL, 1, 4096
    bits, _ = gdn_synth.activations(7, B * T, sh.H, hot="percent")
    w, _ = _make_layer(sh, 7)
    _, ws, lay = nv.gdn_layer_forward(w, bf16_device(bits), B, T)
    torch.cuda.synchronize()
    nv.check_device_error()
    _check_o_quantised_exactly(ws, lay, B * T, sh.Hv * sh.V)


@pytest.mark.parametrize("B,T,block", [(2, 100, False), (3, 1, False), (2, 100, True)])
def test_timed_layer_forward_is_the_same_launches(cuda_dev, B, T, block):
    """gdn_layer_forward_timed (the bench's per-stage timing) runs the same
    launches as gdn_layer_forward: y and the state are bit-identical, and the
    six stage intervals are ordered and add up to the recorded span.  With
    block=True the optional output gate and short convolution are on too (they
    fall inside the gates and quantise-o stages)."""
    sh = gdn_synth.TINY
    bits, _ = gdn_synth.activations(11, B * T, sh.H, hot="percent")
    w, _ = _make_layer(sh, 11)
    if block:
        C = 2 * sh.Hk * sh.K + sh.Hv * sh.V
        w.out_norm = f32_device(1.0 + 0.1 * gdn_synth.gaussian(13, (sh.V,)))
        w.conv_weight = f32_device(0.5 * gdn_synth.gaussian(14, (C, 4)))
        w.conv_width = 4
    S0 = f32_device(gdn_synth.gaussian(12, (B, sh.Hv, sh.K, sh.V), std=0.5))
    x = bf16_device(bits)
    S1, S2 = torch.empty_like(S0), torch.empty_like(S0)
    y1, _, _ = nv.gdn_layer_forward(w, x, B, T, state_in=S0, state_out=S1)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
    y2, _, _ = nv.gdn_layer_forward(w, x, B, T, state_in=S0, state_out=S2, events=evs)
    torch.cuda.synchronize()
    nv.check_device_error()
    assert torch.equal(y1, y2) and torch.equal(S1, S2)
    parts = [evs[i].elapsed_time(evs[i + 1]) for i in range(6)]
    assert all(p >= 0.0 for p in parts)
    assert abs(sum(parts) - evs[0].elapsed_time(evs[6])) <= 1e-3 * max(1.0, sum(parts))
