"""The layer at its full-size configurations on the GPU against the oracle, on a
subset of value heads:
  - the T = 4096 prefill the benchmark times;
  - the T = 32768 long prefill with a state impulse injected at t = 1000;
  - batch-64 decode (256 single-token steps) from a 1024-token prefill.

For each layer call the oracle quantises the same seeded input itself (the
per-tensor scale over every row of that call), forms only the selected heads'
projection columns with a float64 matmul of the dequantised operands, then
applies the gates, the q/k normalisation and the float64 recurrence for those
heads.  Bars: scan output o and final state <= 2e-3 relative Frobenius per head
(the 1e-3 GEMM and 2e-3 scan bars composed, as in the tiny stage-by-stage test)."""
import numpy as np
import pytest
import torch

import gdn_synth
import nvfp4_w4a4_gated_b200 as nv
import oracle
from gpu_util import bf16_device, f32_device, rel_fro

pytestmark = pytest.mark.gpu

TOL = 2e-3
HEADS = (5, 30)   # value heads; GQA key heads 2 and 15


def _make_layer(sh, seed):
    W_in = gdn_synth.weights(seed + 100, sh.n_in, sh.H)
    W_out = gdn_synth.weights(seed + 101, sh.H, sh.Hv * sh.V)
    A_log, dt_bias = gdn_synth.gate_params(seed + 102, sh.Hv)
    dims = nv.GdnDims(sh.Hk, sh.Hv, sh.K, sh.V)
    w = nv.LayerWeights(nv.nvfp4_quantize(f32_device(W_in)), nv.nvfp4_quantize(f32_device(W_out)),
                        f32_device(A_log), f32_device(dt_bias), dims, sh.H)
    W_in_deq = oracle.dequantize(*oracle.quantize(W_in))
    return w, W_in_deq, A_log, dt_bias


def _head_cols(sh, h):
    """Projection columns of value head h: q and k of its key head, v, a, b."""
    hk = h * sh.Hk // sh.Hv
    q = np.arange(hk * sh.K, (hk + 1) * sh.K)
    k = sh.Hk * sh.K + q
    v = 2 * sh.Hk * sh.K + np.arange(h * sh.V, (h + 1) * sh.V)
    a = 2 * sh.Hk * sh.K + 2 * sh.Hv * sh.V + h
    return np.concatenate([q, k, v, [a, a + sh.Hv]])


def _oracle_heads(x, W_in_deq, A_log, dt_bias, sh, B, T, heads, S0=None, rows=None, S0s=None):
    """One layer call's scan for the selected value heads.  x: float32 [B*T, H];
    S0: {h: [b, K, V]} or None; rows: the sequences (batch indices) to compute
    (default all).  Returns {h: (o [b, T, V], S [b, K, V])} for those sequences;
    with S0s (a list of such initial states) a list of those, one per entry."""
    xq = oracle.quantize(x)
    seqs = np.arange(B) if rows is None else np.asarray(rows)
    ridx = (seqs[:, None] * T + np.arange(T)[None, :]).reshape(-1)
    idx = np.concatenate([_head_cols(sh, h) for h in heads])
    Wc = W_in_deq[idx]
    P = np.empty((ridx.size, idx.size))
    for r0 in range(0, ridx.size, 4096):
        rr = ridx[r0:r0 + 4096]
        P[r0:r0 + rr.size] = oracle.dequantize(xq[0][rr], xq[1][rr], xq[2]) @ Wc.T
    nb, K, V = seqs.size, sh.K, sh.V
    starts = [S0] if S0s is None else S0s
    outs = [{} for _ in starts]
    c0 = 0
    for h in heads:
        blk = P[:, c0:c0 + 2 * K + V + 2]
        c0 += 2 * K + V + 2
        g, beta = oracle.gates(blk[:, 2 * K + V:2 * K + V + 1], blk[:, 2 * K + V + 1:], A_log[h:h + 1],
                               dt_bias[h:h + 1])
        qh = oracle.l2norm(blk[:, :K]).reshape(nb, T, 1, K)
        kh = oracle.l2norm(blk[:, K:2 * K]).reshape(nb, T, 1, K)
        for st, out in zip(starts, outs):
            s0 = None if st is None else st[h][:, None]
            o, S = oracle.scan(qh, kh, blk[:, 2 * K:2 * K + V].reshape(nb, T, 1, V), g.reshape(nb, T, 1),
                               beta.reshape(nb, T, 1), S0=s0)
            out[h] = (o[:, :, 0], S[:, 0])
    return outs[0] if S0s is None else outs


def _gpu_o(ws, lay, BT, sh):
    return ws[lay["o"]:lay["o"] + BT * sh.Hv * sh.V * 4].view(torch.float32).view(BT, sh.Hv, sh.V)


def test_prefill_T4096_heads_vs_oracle(cuda_dev):
    """The benchmarked prefill: hidden 5120, 16/32 heads, K = V = 128, B = 1,
    T = 4096, outlier-heavy activations."""
    sh, B, T = gdn_synth.FULL, 1, 4096
    bits, x = gdn_synth.activations(2, B * T, sh.H, hot="percent")
    w, W_in_deq, A_log, dt_bias = _make_layer(sh, 2)
    S_out = torch.empty((B, sh.Hv, sh.K, sh.V), device="cuda")
    _, ws, lay = nv.gdn_layer_forward(w, bf16_device(bits), B, T, state_out=S_out)
    torch.cuda.synchronize()
    nv.check_device_error()
    o = _gpu_o(ws, lay, B * T, sh)
    ref = _oracle_heads(x, W_in_deq, A_log, dt_bias, sh, B, T, HEADS)
    for h in HEADS:
        o_ref, S_ref = ref[h]
        assert rel_fro(o[:, h].cpu().numpy(), o_ref.reshape(B * T, sh.V)) <= TOL
        assert rel_fro(S_out[:, h].cpu().numpy(), S_ref) <= TOL


def test_long_prefill_T32768_with_impulse(cuda_dev):
    """T = 32768 (512 chunks) in two calls: tokens 0..999, then a seeded state
    impulse, then tokens 1000..32767 with the state carried.  Checks o and the
    final state per head, and the impulse response (o with the impulse minus o
    without it) and its decay against the oracle's."""
    sh, B, T, t1 = gdn_synth.FULL, 1, 32768, 1000
    bits, x = gdn_synth.activations(3, B * T, sh.H, hot="percent")
    w, W_in_deq, A_log, dt_bias = _make_layer(sh, 3)
    delta = gdn_synth.gaussian(33, (B, sh.Hv, sh.K, sh.V), std=1.0)
    xb = bf16_device(bits)
    S1 = torch.empty((B, sh.Hv, sh.K, sh.V), device="cuda")
    nv.gdn_layer_forward(w, xb[:t1].contiguous(), B, t1, state_out=S1)
    runs = {}
    for name, d in (("impulse", delta), ("none", None)):
        S_in = S1 + (f32_device(delta) if d is not None else 0.0)
        S_end = torch.empty_like(S1)
        _, ws, lay = nv.gdn_layer_forward(w, xb[t1:].contiguous(), B, T - t1, state_in=S_in, state_out=S_end)
        torch.cuda.synchronize()
        runs[name] = (_gpu_o(ws, lay, B * (T - t1), sh)[:, list(HEADS)].cpu().numpy(), S_end[:, list(HEADS)].cpu().numpy())
        del ws
    nv.check_device_error()
    r1 = _oracle_heads(x[:t1], W_in_deq, A_log, dt_bias, sh, B, t1, HEADS)
    starts = [{h: r1[h][1] + delta[:, h] for h in HEADS}, {h: r1[h][1] for h in HEADS}]
    r_imp, r_none = _oracle_heads(x[t1:], W_in_deq, A_log, dt_bias, sh, B, T - t1, HEADS, S0s=starts)
    ref = {"impulse": r_imp, "none": r_none}
    for j, h in enumerate(HEADS):
        o_g, S_g = runs["impulse"][0][:, j], runs["impulse"][1][:, j]
        o_r, S_r = ref["impulse"][h]
        assert rel_fro(o_g, o_r.reshape(-1, sh.V)) <= TOL
        assert rel_fro(S_g, S_r) <= TOL
        # impulse response over the first chunk after t1, and what is left of it at the end
        resp_g = runs["impulse"][0][:, j] - runs["none"][0][:, j]
        resp_r = (ref["impulse"][h][0] - ref["none"][h][0]).reshape(-1, sh.V)
        assert np.linalg.norm(resp_r[:64]) > 0
        assert rel_fro(resp_g[:64], resp_r[:64]) <= 1e-2
        late_r = np.linalg.norm(resp_r[-64:])
        assert np.linalg.norm(resp_g[-64:]) <= late_r + 1e-3 * np.linalg.norm(resp_r[:64])


def test_decode_B64_from_prefill(cuda_dev):
    """Batch-64 decode: a 1024-token prefill of N(0,1) inputs, then 256
    single-token steps with the states carried.  o of every step and the final
    states are checked for two sequences and two value heads."""
    sh, B, T0, steps = gdn_synth.FULL, 64, 1024, 256
    seqs = (0, 41)
    w, W_in_deq, A_log, dt_bias = _make_layer(sh, 4)
    bits0, x0 = gdn_synth.activations(4, B * T0, sh.H, hot="none")
    S = torch.empty((B, sh.Hv, sh.K, sh.V), device="cuda")
    nv.gdn_layer_forward(w, bf16_device(bits0), B, T0, state_out=S)
    ref = _oracle_heads(x0, W_in_deq, A_log, dt_bias, sh, B, T0, HEADS, rows=seqs)
    S_ref = {h: ref[h][1] for h in HEADS}
    o_gpu, o_ref = [], []
    for t in range(steps):
        bits, x = gdn_synth.activations(1000 + t, B, sh.H, hot="none")
        _, ws, lay = nv.gdn_layer_forward(w, bf16_device(bits), B, 1, state_in=S, state_out=S)
        o_gpu.append(_gpu_o(ws, lay, B, sh)[list(seqs)][:, list(HEADS)].cpu().numpy())
        r = _oracle_heads(x, W_in_deq, A_log, dt_bias, sh, B, 1, HEADS, S0=S_ref, rows=seqs)
        S_ref = {h: r[h][1] for h in HEADS}
        o_ref.append(np.stack([r[h][0][:, 0] for h in HEADS], axis=1))
    torch.cuda.synchronize()
    nv.check_device_error()
    o_gpu, o_ref = np.stack(o_gpu), np.stack(o_ref)
    S_gpu = S[list(seqs)][:, list(HEADS)].cpu().numpy()
    for j, h in enumerate(HEADS):
        assert rel_fro(o_gpu[:, :, j], o_ref[:, :, j]) <= TOL
        assert rel_fro(S_gpu[:, j], S_ref[h]) <= TOL
