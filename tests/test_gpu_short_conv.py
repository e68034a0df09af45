"""Optional short causal convolution (reading C1: width-W depthwise causal
convolution + SiLU on the q|k|v channels, carried state of the last W-1
inputs) on the GPU against the oracle: the standalone call and the layer with
the convolution weight set.

float32 fma against the oracle's float64: 1e-5 relative per element (plus 1e-6
of the channel scale).  The new state is a copy of inputs: exact."""
import numpy as np
import pytest
import torch

import gdn_synth
import nvfp4_w4a4_gated_b200 as nv
import oracle
from gpu_util import bf16_device, f32_device, rel_fro

pytestmark = pytest.mark.gpu


def _close(got, ref):
    scale = np.abs(ref).max() + 1e-30
    assert np.all(np.abs(got - ref) <= 1e-5 * np.abs(ref) + 1e-6 * scale)


@pytest.mark.parametrize("W", [2, 3, 4])
@pytest.mark.parametrize("with_state", [False, True])
@pytest.mark.parametrize("C", [300, 301])   # 301: no 16-byte access, the one-channel-per-thread kernel
def test_short_conv_matches_oracle(cuda_dev, W, with_state, C):
    B, T, extra = 2, 45, 12                  # ragged: tokens past one 32-token block, channels past 2 x 128
    xbig = gdn_synth.gaussian(40 + W, (B * T, C + extra), std=2.0)
    w = gdn_synth.gaussian(41 + W, (C, W), std=0.7)
    s0 = gdn_synth.gaussian(42 + W, (B, C, W - 1), std=2.0) if with_state else None
    x_d = f32_device(xbig)
    s_in = f32_device(s0) if with_state else None
    s_out = torch.empty((B, C, W - 1), device="cuda")
    out = nv.gdn_short_conv(x_d, f32_device(w), B, T, state_in=s_in, state_out=s_out)
    torch.cuda.synchronize()
    nv.check_device_error()
    ref, ref_state = oracle.short_conv(xbig[:, :C], w, B, T, state_in=s0, return_state=True)
    _close(out.cpu().numpy(), ref)
    assert np.array_equal(s_out.cpu().numpy(), ref_state.astype(np.float32))


def test_short_conv_token_by_token_equals_whole_sequence(cuda_dev):
    """Decode: T single-token calls with the state updated in place give the same
    outputs, bit for bit, as one call over the T tokens."""
    B, T, C, W = 3, 9, 256, 4
    x = f32_device(gdn_synth.gaussian(50, (B, T, C), std=1.0))
    w = f32_device(gdn_synth.gaussian(51, (C, W), std=0.7))
    whole = nv.gdn_short_conv(x.view(B * T, C), w, B, T).view(B, T, C)
    state = torch.zeros((B, C, W - 1), device="cuda")
    steps = []
    for t in range(T):
        xt = x[:, t].contiguous()
        steps.append(nv.gdn_short_conv(xt, w, B, 1, state_in=state, state_out=state))
    torch.cuda.synchronize()
    nv.check_device_error()
    assert torch.equal(torch.stack(steps, 1), whole)


@pytest.mark.parametrize("B,T", [(1, 64), (2, 100)])
def test_layer_with_short_conv(cuda_dev, B, T):
    """The layer with the convolution: the convolved q|k|v against the oracle
    convolution of the GPU's own projection; the scan output o and final state
    against the oracle recurrence on those inputs (2e-3); the new convolution
    state is the projection's last W-1 q|k|v rows.  Then one decode step with both
    states carried matches the oracle on the same inputs."""
    sh = gdn_synth.TINY
    C, W = 2 * sh.Hk * sh.K + sh.Hv * sh.V, 4
    W_in = gdn_synth.weights(130, sh.n_in, sh.H)
    W_out = gdn_synth.weights(131, sh.H, sh.Hv * sh.V)
    A_log, dt_bias = gdn_synth.gate_params(132, sh.Hv)
    conv_w = gdn_synth.gaussian(133, (C, W), std=0.5)
    dims = nv.GdnDims(sh.Hk, sh.Hv, sh.K, sh.V)
    w = nv.LayerWeights(nv.nvfp4_quantize(f32_device(W_in)), nv.nvfp4_quantize(f32_device(W_out)),
                        f32_device(A_log), f32_device(dt_bias), dims, sh.H, None, f32_device(conv_w), W)
    bits, _ = gdn_synth.activations(134 + B, B * T, sh.H, hot="fixed")
    S = torch.empty((B, sh.Hv, sh.K, sh.V), device="cuda")
    cs = torch.empty((B, C, W - 1), device="cuda")
    y, ws, lay = nv.gdn_layer_forward(w, bf16_device(bits), B, T, state_out=S, conv_state_out=cs)
    torch.cuda.synchronize()
    nv.check_device_error()
    BT, ldp = B * T, (sh.n_in + 3) // 4 * 4

    def view(name, nbytes):
        return ws[lay[name]:lay[name] + nbytes].view(torch.float32).cpu().numpy()

    P = view("proj", BT * ldp * 4).reshape(BT, ldp)[:, : sh.n_in]
    qkv = view("qkv_conv", BT * C * 4).reshape(BT, C)
    ref_qkv, ref_cs = oracle.short_conv(P[:, :C], conv_w, B, T, return_state=True)
    _close(qkv, ref_qkv)
    assert np.array_equal(cs.cpu().numpy(), ref_cs.astype(np.float32))
    # the scan on the convolved q|k|v and the raw a|b
    q, k, v, _, a, b = oracle.split_projection(np.concatenate([ref_qkv, P[:, C:]], axis=1), sh.Hk, sh.Hv, sh.K, sh.V)
    g, beta = oracle.gates(a, b, A_log, dt_bias)
    o_ref, S_ref = oracle.scan(oracle.l2norm(q.reshape(B, T, sh.Hk, sh.K)), oracle.l2norm(k.reshape(B, T, sh.Hk, sh.K)),
                               v.reshape(B, T, sh.Hv, sh.V), g.reshape(B, T, sh.Hv), beta.reshape(B, T, sh.Hv))
    o = view("o", BT * sh.Hv * sh.V * 4).reshape(B, T, sh.Hv, sh.V)
    assert rel_fro(o, o_ref) <= 2e-3
    assert rel_fro(S.cpu().numpy(), S_ref) <= 2e-3
    # one decode step with both states carried in place
    bits1, _ = gdn_synth.activations(140 + B, B, sh.H, hot="none")
    y1, ws1, lay1 = nv.gdn_layer_forward(w, bf16_device(bits1), B, 1, state_in=S, state_out=S, conv_state_in=cs,
                                         conv_state_out=cs)
    torch.cuda.synchronize()
    nv.check_device_error()
    P1 = ws1[lay1["proj"]:lay1["proj"] + B * ldp * 4].view(torch.float32).cpu().numpy().reshape(B, ldp)[:, : sh.n_in]
    ref_qkv1, ref_cs1 = oracle.short_conv(P1[:, :C], conv_w, B, 1, state_in=ref_cs, return_state=True)
    qkv1 = ws1[lay1["qkv_conv"]:lay1["qkv_conv"] + B * C * 4].view(torch.float32).cpu().numpy().reshape(B, C)
    _close(qkv1, ref_qkv1)
    assert np.array_equal(cs.cpu().numpy(), ref_cs1.astype(np.float32))
    q, k, v, _, a, b = oracle.split_projection(np.concatenate([ref_qkv1, P1[:, C:]], axis=1), sh.Hk, sh.Hv, sh.K, sh.V)
    g, beta = oracle.gates(a, b, A_log, dt_bias)
    o1_ref, S1_ref = oracle.scan(oracle.l2norm(q.reshape(B, 1, sh.Hk, sh.K)), oracle.l2norm(k.reshape(B, 1, sh.Hk, sh.K)),
                                 v.reshape(B, 1, sh.Hv, sh.V), g.reshape(B, 1, sh.Hv), beta.reshape(B, 1, sh.Hv),
                                 S0=S_ref)
    o1 = ws1[lay1["o"]:lay1["o"] + B * sh.Hv * sh.V * 4].view(torch.float32).cpu().numpy().reshape(B, 1, sh.Hv, sh.V)
    assert rel_fro(o1, o1_ref) <= 2e-3
    assert rel_fro(S.cpu().numpy(), S1_ref) <= 2e-3
