"""The sequence-split layer on one GPU (seqpar.segmented_layer: the steps of
sequence_parallel_layer with the spans in order and the maximum of their amax
words in place of the all-reduce) against the oracle's whole-sequence layer.
The quantised x of every span is the whole tensor's rows bit for bit; o, the
o codes, y and the final state are held to the stage-wise bars of the layer
tests."""
import numpy as np
import pytest
import torch

import gdn_synth
import nvfp4_w4a4_gated_b200 as nv
import oracle
from gpu_util import bf16_device, f32_device, rel_fro
from nvfp4_w4a4_gated_b200.seqpar import segmented_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("form", [nv.FORM_PAGES, nv.FORM_STANDARD])
def test_segmented_layer_matches_the_whole_layer(cuda_dev, form):
    sh, B, T = gdn_synth.TINY, 2, 100
    bounds = [0, 37, 38, 100]
    bits, x = gdn_synth.activations(20, B * T, sh.H, hot="fixed")
    W_in = gdn_synth.weights(21, sh.n_in, sh.H)
    W_out = gdn_synth.weights(22, sh.H, sh.Hv * sh.V)
    A_log, dt_bias = gdn_synth.gate_params(23, sh.Hv)
    S0 = gdn_synth.gaussian(24, (B, sh.Hv, sh.K, sh.V), std=0.5)
    dims = nv.GdnDims(sh.Hk, sh.Hv, sh.K, sh.V)
    w = nv.LayerWeights(nv.nvfp4_quantize(f32_device(W_in)), nv.nvfp4_quantize(f32_device(W_out)), f32_device(A_log),
                        f32_device(dt_bias), dims, sh.H)
    xb = bf16_device(bits).view(B, T, sh.H)
    xs = [(xb[:, a:e].reshape(B * (e - a), sh.H).contiguous(), e - a) for a, e in zip(bounds, bounds[1:])]
    ys, xqs, oqs, S = segmented_layer(w, xs, B, form=form, state_in=f32_device(S0))
    torch.cuda.synchronize()
    nv.check_device_error()
    ref = oracle.layer_forward(x, oracle.quantize(W_in), oracle.quantize(W_out), A_log, dt_bias, B, T, sh.Hk, sh.Hv,
                               sh.K, sh.V, form=form, S0=S0, stages=True)
    HvV = sh.Hv * sh.V
    rows = lambda m, a, e: np.ascontiguousarray(m.reshape(B, T, -1)[:, a:e].reshape(B * (e - a), -1))
    y_all, flips = [], []
    for (a, e), xq, oq, y in zip(zip(bounds, bounds[1:]), xqs, oqs, ys):
        n = B * (e - a)
        assert np.array_equal(xq.codes.cpu().numpy(), rows(ref["xq"][0], a, e))
        assert np.array_equal(xq.sf.cpu().numpy(), oracle.sf_linear_to_mma(rows(ref["xq"][1], a, e), n, sh.H))
        assert np.float32(xq.scale.cpu().numpy()[0]) == np.float32(ref["xq"][2])
        flips.append(np.mean(oq.codes.cpu().numpy() != rows(ref["oq"][0], a, e)))
        y_all.append(y.cpu().numpy().reshape(B, e - a, sh.H))
    # o itself: the codes carry it; both sides' o scales agree to the scan bar
    assert abs(float(oqs[0].scale.cpu().numpy()[0]) / float(ref["oq"][2]) - 1.0) <= 2e-3
    assert all(float(oq.scale.cpu().numpy()[0]) == float(oqs[0].scale.cpu().numpy()[0]) for oq in oqs)
    flipped = float(np.mean(flips))
    assert flipped < 0.02
    y_got = np.concatenate(y_all, axis=1).reshape(B * T, sh.H)
    assert rel_fro(y_got, ref["y"]) <= max(2e-2, 0.5 * np.sqrt(flipped))
    assert rel_fro(S.cpu().numpy(), ref["S"]) <= 2e-3
