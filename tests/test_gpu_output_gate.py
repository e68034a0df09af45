"""Optional output gate (reading O1: G = RMSNorm(o) * w * SiLU(z) per token and
value head) on the GPU against the oracle: the standalone call, and the layer
with the gate weight set, stage by stage downstream of the scan.

The gate is float32 arithmetic against the oracle's float64: bar 1e-5 relative
per element (on top of an absolute 1e-6 of the row scale).  The quantisation of
the GPU's gated output is bit-exact against the oracle's quantisation of the
same values, and y is held to the GEMM bar (1e-3) against the oracle's float64
product of those codes."""
import numpy as np
import pytest
import torch

import gdn_synth
import nvfp4_w4a4_gated_b200 as nv
import oracle
from gpu_util import bf16_device, f32_device, rel_fro

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("V", [64, 128])
@pytest.mark.parametrize("inplace", [False, True])
def test_output_gate_matches_oracle(cuda_dev, V, inplace):
    n, Hv, ld_extra = 203, 3, 12
    o = gdn_synth.gaussian(20 + V, (n, Hv, V), std=3.0)
    o[5, 1] = 0.0                                   # an all-zero row
    zbig = gdn_synth.gaussian(21 + V, (n, Hv * V + ld_extra), std=2.0)
    w = gdn_synth.gaussian(22 + V, (V,), std=1.0)
    o_d, z_d, w_d = f32_device(o), f32_device(zbig), f32_device(w)
    amax = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = nv.gdn_output_gate(o_d, z_d[:, : Hv * V + ld_extra], w_d, out=o_d if inplace else None, amax_word=amax)
    torch.cuda.synchronize()
    nv.check_device_error()
    got = out.cpu().numpy()
    ref = oracle.output_gate(o, zbig[:, : Hv * V].reshape(n, Hv, V), w)
    scale = np.abs(ref).max(axis=-1, keepdims=True)
    assert np.all(np.abs(got - ref) <= 1e-5 * np.abs(ref) + 1e-6 * scale)
    assert np.all(got[5, 1] == 0.0)
    assert amax.cpu().numpy().view(np.float32)[0] == np.abs(got).max()


def _layer(seed, with_gate):
    sh = gdn_synth.TINY
    W_in = gdn_synth.weights(seed + 100, sh.n_in, sh.H)
    W_out = gdn_synth.weights(seed + 101, sh.H, sh.Hv * sh.V)
    A_log, dt_bias = gdn_synth.gate_params(seed + 102, sh.Hv)
    w_norm = gdn_synth.gaussian(seed + 103, (sh.V,), std=1.0) if with_gate else None
    dims = nv.GdnDims(sh.Hk, sh.Hv, sh.K, sh.V)
    w = nv.LayerWeights(nv.nvfp4_quantize(f32_device(W_in)), nv.nvfp4_quantize(f32_device(W_out)),
                        f32_device(A_log), f32_device(dt_bias), dims, sh.H,
                        None if w_norm is None else f32_device(w_norm))
    return sh, w, W_out, w_norm


@pytest.mark.parametrize("B,T", [(1, 64), (2, 100), (64, 1)])
def test_layer_with_output_gate(cuda_dev, B, T):
    sh, w, W_out, w_norm = _layer(7, True)
    bits, _ = gdn_synth.activations(70 + B, B * T, sh.H, hot="fixed")
    y, ws, lay = nv.gdn_layer_forward(w, bf16_device(bits), B, T)
    torch.cuda.synchronize()
    nv.check_device_error()
    BT, HvV = B * T, sh.Hv * sh.V
    ldp = (sh.n_in + 3) // 4 * 4

    def view(name, nbytes, dtype):
        return ws[lay[name]:lay[name] + nbytes].view(dtype).cpu().numpy()

    o = view("o", BT * HvV * 4, torch.float32).reshape(BT, sh.Hv, sh.V)
    P = view("proj", BT * ldp * 4, torch.float32).reshape(BT, ldp)[:, : sh.n_in]
    z = oracle.split_projection(P, sh.Hk, sh.Hv, sh.K, sh.V)[3].reshape(BT, sh.Hv, sh.V)
    G = view("o_gated", BT * HvV * 4, torch.float32).reshape(BT, sh.Hv, sh.V)
    G_ref = oracle.output_gate(o, z, w_norm)
    scale = np.abs(G_ref).max(axis=-1, keepdims=True)
    assert np.all(np.abs(G - G_ref) <= 1e-5 * np.abs(G_ref) + 1e-6 * scale)
    # out_proj quantised the gated output: codes and scales bit-exact, y at the GEMM bar
    codes, sf, S = oracle.quantize(G.reshape(BT, HvV))
    assert np.array_equal(view("o_codes", BT * HvV // 2, torch.uint8).reshape(BT, HvV // 2), codes)
    assert np.array_equal(view("o_sf", nv.lib().nvfp4_sf_bytes(BT, HvV), torch.uint8),
                          oracle.sf_linear_to_mma(sf, BT, HvV))
    ref_y = oracle.w4a4_gemm((codes, sf, S), oracle.quantize(W_out))
    assert rel_fro(y.cpu().numpy(), ref_y) <= 1e-3


def test_layer_gate_changes_only_the_output_path(cuda_dev):
    """Same inputs with and without the gate weight: everything up to the scan
    output is identical; y differs."""
    bits, _ = gdn_synth.activations(80, 64, gdn_synth.TINY.H, hot="fixed")
    sh, w0, _, _ = _layer(8, False)
    _, w1, _, _ = _layer(8, True)
    y0, ws0, lay0 = nv.gdn_layer_forward(w0, bf16_device(bits), 1, 64)
    y1, ws1, lay1 = nv.gdn_layer_forward(w1, bf16_device(bits), 1, 64)
    torch.cuda.synchronize()
    nv.check_device_error()
    n = 64 * sh.Hv * sh.V * 4
    assert torch.equal(ws0[lay0["o"]:lay0["o"] + n], ws1[lay1["o"]:lay1["o"] + n])
    assert not torch.equal(y0, y1)
