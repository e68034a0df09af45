"""Pins of the CPU oracle against facts fixed outside it: the pages' printed
format facts and bounds, closed forms, library routines (torch float8,
numpy) and brute force on tiny inputs.  CPU only."""
import math

import numpy as np
import pytest
import torch

import oracle
import gdn_synth
from conftest import read_golden

E2M1_MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


# ----------------------------------------------------------------- formats --
def test_e2m1_grid_matches_golden():
    for code_s, val_s in read_golden("e2m1_grid.txt"):
        code, val = int(code_s, 16), float(val_s)
        got = oracle.e2m1_decode(code)
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)
        assert oracle.e2m1_encode(val) == code


def _e2m1_bruteforce(y):
    """Nearest grid magnitude; on a tie the one with an even mantissa bit
    (code index even); above 6 saturate."""
    a = abs(y)
    dists = [abs(a - m) for m in E2M1_MAGS]
    best = min(dists)
    cands = [i for i, d in enumerate(dists) if d == best]
    if len(cands) > 1:
        cands = [i for i in cands if i % 2 == 0]
    idx = cands[0]
    if a >= 6.0:
        idx = 7
    return (8 if math.copysign(1, y) < 0 else 0) | idx


def test_e2m1_rounding_bruteforce():
    ys = list(np.linspace(-8, 8, 4001, dtype=np.float32))
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0]
    for t in ties:
        for s in (1, -1):
            ys += [np.float32(s * t), np.nextafter(np.float32(s * t), np.float32(0)),
                   np.nextafter(np.float32(s * t), np.float32(s * 100))]
    ys += [np.float32(-0.0), np.float32(1e-30), np.float32(-1e-30), np.float32(1e30), np.float32(-1e30)]
    for y in ys:
        assert oracle.e2m1_encode(float(y)) == _e2m1_bruteforce(float(y)), y


def test_e2m1_ties_spot_values():
    # ties to the even mantissa: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    want = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0, 6.5: 6.0, 100.0: 6.0}
    for y, v in want.items():
        assert oracle.e2m1_decode(oracle.e2m1_encode(y)) == v


def test_e4m3_decode_matches_torch_float8():
    bits = torch.arange(256, dtype=torch.uint8)
    ref = bits.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for b in range(256):
        got = oracle.e4m3_decode(b)
        if np.isnan(ref[b]):
            assert np.isnan(got)
        else:
            assert got == ref[b], (b, got, ref[b])


def test_e4m3_encode_matches_torch_float8():
    g = gdn_synth.rng(123)
    vals = np.exp(g.uniform(np.log(2.0 ** -12), np.log(447.0), 20000)).astype(np.float32)
    # exact ties between neighbouring E4M3 values and the subnormal range
    reps = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mids = ((reps[1:] + reps[:-1]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, reps.astype(np.float32), np.float32([2.0 ** -10, 2.0 ** -11, 3e-3])])
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, r in zip(vals, ref):
        assert oracle.e4m3_encode(float(v)) == int(r), (v, oracle.e4m3_encode(float(v)), r)


def test_e4m3_encode_saturates():
    for v in (448.0, 449.0, 464.0, 500.0, 1e6, 3e38):
        assert oracle.e4m3_encode(v) == 0x7E
    assert oracle.e4m3_encode(0.0) == 0


# --------------------------------------------------------------- quantiser --
def test_roundtrip_exact_on_scaled_grid():
    """Values already of the form code * E4M3 * S with S a power of two, every
    block containing a +-6 and one block at scale 448, come back bit-exactly."""
    g = gdn_synth.rng(7)
    rows, cols = 8, 64
    S = np.float32(2.0 ** -3)
    nb = cols // 16
    sbs = g.integers(0x08, 0x7F, size=(rows, nb)).astype(np.uint8)   # normal E4M3 scales, no NaN
    sbs[3, 2] = 0x7E                                                  # 448
    codes_lin = g.integers(0, 16, size=(rows, cols)).astype(np.uint8)
    codes_lin[:, ::16] = 0x7                                          # a +6 in every block
    codes_lin[:, 5::16] = 0xF                                         # and a -6
    vals = np.array([[float(v) for v in row] for row in np.vectorize(oracle.e2m1_decode)(codes_lin)])
    scl = np.vectorize(oracle.e4m3_decode)(sbs)
    x = (vals * np.repeat(scl, 16, axis=1) * float(S)).astype(np.float32)
    assert np.all(x.astype(np.float64) == vals * np.repeat(scl, 16, axis=1) * float(S))
    codes, sf, S2 = oracle.quantize(x)
    assert S2 == S
    assert np.array_equal(sf, sbs)
    packed = (codes_lin[:, 0::2] | (codes_lin[:, 1::2] << 4)).astype(np.uint8)
    # -0 codes cannot arise here except for code 8 itself, which decodes to -0 and re-encodes as 8
    assert np.array_equal(codes, packed)


def test_block_bound_max_over_rms():
    rows = {r[0]: float(r[1]) for r in read_golden("block_bound.txt")}
    bs, bound = int(rows["block_size"]), rows["max_over_rms_bound"]
    assert bound == math.sqrt(bs)
    _, x = gdn_synth.activations(11, 64, 512, hot="percent")
    codes, sf, S = oracle.quantize(x)
    xd = oracle.dequantize(codes, sf, S)
    for arr in (x.astype(np.float64), xd):
        blk = arr.reshape(-1, bs)
        nz = np.any(blk != 0, axis=1)
        ratio = np.abs(blk[nz]).max(1) / np.sqrt((blk[nz] ** 2).mean(1))
        assert np.all(ratio <= bound * (1 + 1e-12))
    # one-hot blocks reach the bound exactly, before and after quantisation
    oh = np.zeros((4, 64), np.float32)
    oh[np.arange(4), [0, 17, 34, 63]] = [1.0, -2.5, 3.0, 0.75]
    c, s, S = oracle.quantize(oh)
    d = oracle.dequantize(c, s, S).reshape(-1, bs)
    nz = np.any(d != 0, axis=1)
    ratio = np.abs(d[nz]).max(1) / np.sqrt((d[nz] ** 2).mean(1))
    assert np.allclose(ratio, bound, rtol=0, atol=1e-12)


def test_outlier_localised_to_its_block():
    rows = {r[0]: float(r[1]) for r in read_golden("block_bound.txt")}
    nnb = int(rows["neighbours_degraded"])
    _, x = gdn_synth.activations(12, 16, 256, hot="none")
    c0, s0, S0 = oracle.quantize(x)
    # (i) an outlier that does not raise the tensor amax changes only its own block
    x1 = x.copy()
    amax = np.abs(x).max()
    r, col = 5, 37
    x1[r, col] = np.float32(amax * 0.99)
    c1, s1, S1 = oracle.quantize(x1)
    assert S1 == S0
    blk = col // 16
    diff_sf = np.argwhere(s1 != s0)
    assert all(tuple(d) == (r, blk) for d in diff_sf)
    diff_c = np.argwhere(c1 != c0)
    assert all(d[0] == r and d[1] // 8 == blk for d in diff_c)
    # (ii) an outlier 100x the amax: its block's other 15 values collapse, the rest keep
    # their usual error level
    x2 = x.copy()
    x2[r, col] = np.float32(amax * 100)
    c2, s2, S2 = oracle.quantize(x2)
    d2 = oracle.dequantize(c2, s2, S2)
    err = np.abs(d2 - x2)
    hot = np.zeros_like(x2, bool)
    hot[r, blk * 16:(blk + 1) * 16] = True
    hot[r, col] = False
    assert hot.sum() == nnb
    rel_hot = np.linalg.norm(err[hot]) / np.linalg.norm(x2[hot])
    rel_rest = np.linalg.norm(err[~hot & (np.arange(256)[None] != col)]) / np.linalg.norm(x2[~hot & (np.arange(256)[None] != col)])
    assert rel_hot > 0.5
    assert rel_rest < 0.2


def test_zero_and_tiny_tensors():
    x = np.zeros((4, 32), np.float32)
    c, s, S = oracle.quantize(x)
    assert S == 1.0 and not c.any() and not s.any()
    x[1, 3] = 1e-35
    c, s, S = oracle.quantize(x)
    assert S == 1.0 and not c.any() and not s.any()
    x = np.full((2, 16), -1e-3, np.float32)
    x[0, 0] = 1.0
    c, s, S = oracle.quantize(x)
    # row 1 is 1e-3 of the amax: scale 1e-3*448 ~ 0.45 -> representable, codes = -6 -> 0xF
    assert s[1, 0] != 0 and np.all(c[1] == 0xFF)


def test_sf_layout_is_the_atom_permutation():
    rows, cols = 300, 512
    g = gdn_synth.rng(5)
    sf = g.integers(0, 256, size=(rows, cols // 16)).astype(np.uint8)
    out = oracle.sf_linear_to_mma(sf, rows, cols)
    # independent construction: pad, then reshape [rb, 4 (row/32), 32 (row%32), kb, 4] and
    # reorder to [rb, kb, 32, 4, 4]
    prow = (rows + 127) // 128 * 128
    pad = np.zeros((prow, cols // 16), np.uint8)
    pad[:rows] = sf
    t = pad.reshape(prow // 128, 4, 32, cols // 64, 4).transpose(0, 3, 2, 1, 4)
    assert np.array_equal(out, t.reshape(-1))


# -------------------------------------------------------------------- GEMM --
def test_dequantize_is_code_times_scale_times_S():
    _, x = gdn_synth.activations(13, 8, 64, hot="fixed")
    c, s, S = oracle.quantize(x)
    d = oracle.dequantize(c, s, S)
    grid = {int(a, 16): float(b) for a, b in read_golden("e2m1_grid.txt")}
    sfv = torch.from_numpy(s.copy()).view(torch.float8_e4m3fn).double().numpy()
    for r in range(8):
        for col in range(64):
            byte = c[r, col // 2]
            code = (byte >> 4) if col % 2 else (byte & 15)
            assert d[r, col] == grid[int(code)] * sfv[r, col // 16] * float(S)


def test_gemm_matches_numpy_and_bruteforce():
    g = gdn_synth.rng(9)
    A = g.standard_normal((7, 48))
    B = g.standard_normal((5, 48))
    C = oracle.gemm_nt(A, B)
    assert np.allclose(C, A @ B.T, rtol=1e-13, atol=1e-13)
    for i in range(7):
        for j in range(5):
            assert abs(C[i, j] - sum(A[i, k] * B[j, k] for k in range(48))) < 1e-12


def test_harmonised_fused_gemm_equals_per_slice():
    """One weight scale for the fused tensor: the fused GEMM equals the
    concatenation of per-slice GEMMs run under that shared scale; with
    per-module scales applied through one fused scale, slice m is off by
    S_0 / S_m (the mismatch the pages repair; review page sec.6, abstract)."""
    sl, gain = (32, 32, 64), (1.0, 4.0, 2.0)
    W = gdn_synth.weights(21, sum(sl), 128, slice_rows=sl, slice_gain=gain)
    _, x = gdn_synth.activations(22, 16, 128, hot="fixed")
    xq = oracle.quantize(x)
    Wq = oracle.quantize(W)                       # harmonised: one amax over the fused tensor
    fused = oracle.w4a4_gemm(xq, Wq)
    r0, parts, own = 0, [], []
    for n in sl:
        part = oracle.quantize(W[r0:r0 + n], S=Wq[2])
        assert np.array_equal(part[0], Wq[0][r0:r0 + n]) and np.array_equal(part[1], Wq[1][r0:r0 + n])
        parts.append(oracle.w4a4_gemm(xq, part))
        own.append(oracle.quantize(W[r0:r0 + n]))
        r0 += n
    assert np.array_equal(fused, np.concatenate(parts, axis=1))
    # negative control: per-module codes/scales served with module 0's global scale
    S0 = own[0][2]
    bad = np.concatenate([oracle.w4a4_gemm(xq, (c, s, S0)) for c, s, _ in own], axis=1)
    good = np.concatenate([oracle.w4a4_gemm(xq, o) for o in own], axis=1)
    r0 = 0
    for (c, s, Sm), n in zip(own, sl):
        ratio = float(S0) / float(Sm)
        assert np.allclose(bad[:, r0:r0 + n], good[:, r0:r0 + n] * ratio, rtol=1e-12, atol=0)
        r0 += n
    rel = np.linalg.norm(bad[:, 32:64] - good[:, 32:64]) / np.linalg.norm(good[:, 32:64])
    assert rel > 0.5


# ------------------------------------------------------------------- gates --
def test_softplus_closed_forms():
    assert abs(oracle.softplus(0.0) - math.log(2.0)) < 1e-15
    for u in (-30.0, -3.0, -0.5, 0.7, 5.0, 40.0):
        assert abs(oracle.softplus(u) - float(np.logaddexp(0.0, u))) <= 1e-15 * max(1, abs(u))
    assert oracle.softplus(800.0) == 800.0


def test_softplus_limits():
    """softplus(u) -> u as u -> +inf (the log1p term is below the last bit of u
    once e^-u < 2^-53 u) and -> e^u as u -> -inf."""
    for u in (40.0, 60.0, 200.0):
        assert oracle.softplus(u) == u
    for u in (-40.0, -60.0, -200.0):
        assert abs(oracle.softplus(u) / math.exp(u) - 1.0) < 1e-15


# The gate heads below: per-head A_log and dt_bias all different and non-zero, so
# that a dropped or swapped parameter moves every closed form.
_A_LOG = np.array([math.log(1.5), math.log(4.0), math.log(16.0), -0.75])
_DT_BIAS = np.array([0.3, -1.2, 2.0, -0.45])


def test_gates_closed_form_at_zero_softplus_argument():
    """Eq.(1) at a + dt_bias = 0: softplus(0) = ln 2, so g = -e^{A_log} ln 2
    per head (review page, paper sec.2)."""
    a = np.tile(-_DT_BIAS, (3, 1))
    g, _ = oracle.gates(a, np.zeros_like(a), _A_LOG, _DT_BIAS)
    want = -np.exp(_A_LOG) * math.log(2.0)
    assert np.allclose(g, np.tile(want, (3, 1)), rtol=1e-15, atol=0)


def test_gates_closed_form_at_unit_softplus():
    """a + dt_bias = ln(e - 1) gives softplus = ln(1 + e - 1) = 1, so g = -e^{A_log}
    and the decay alpha = exp(-e^{A_log}); at A_log = ln 4 that is e^-4."""
    a = np.tile(math.log(math.e - 1.0) - _DT_BIAS, (2, 1))
    g, _ = oracle.gates(a, np.zeros_like(a), _A_LOG, _DT_BIAS)
    assert np.allclose(g, np.tile(-np.exp(_A_LOG), (2, 1)), rtol=1e-14, atol=0)
    assert abs(math.exp(g[0, 1]) - math.exp(-4.0)) < 1e-15


def test_beta_closed_forms():
    """beta = sigmoid(b): 1/2 at b = 0, 3/4 at b = ln 3, 1/4 at b = -ln 3
    (1 / (1 + 1/3) and 1 / (1 + 3)), whatever A_log and dt_bias are."""
    l3 = math.log(3.0)
    b = np.array([[0.0, l3, -l3, 0.0], [l3, -l3, 0.0, l3]])
    _, beta = oracle.gates(np.zeros_like(b), b, _A_LOG, _DT_BIAS)
    want = np.array([[0.5, 0.75, 0.25, 0.5], [0.75, 0.25, 0.5, 0.75]])
    assert np.allclose(beta, want, rtol=1e-15, atol=0)


def test_gates_monotone_and_in_range():
    """alpha = e^g lies in (0, 1) and strictly decreases as a grows (a larger
    step forgets more); beta lies in (0, 1) and strictly increases with b."""
    u = np.linspace(-8.0, 8.0, 161)
    a = np.repeat(u[:, None], 4, axis=1)
    g, beta = oracle.gates(a, a, _A_LOG, _DT_BIAS)
    alpha = np.exp(g)
    assert np.all((alpha > 0) & (alpha < 1)) and np.all((beta > 0) & (beta < 1))
    assert np.all(np.diff(alpha, axis=0) < 0)
    assert np.all(np.diff(beta, axis=0) > 0)


def test_gates_heads_are_independent():
    """Head h reads only A_log[h] and dt_bias[h]: permuting the heads' parameters
    together with the columns of a and b permutes the outputs."""
    g0 = gdn_synth.rng(31)
    a = g0.standard_normal((20, 4)) * 3
    b = g0.standard_normal((20, 4)) * 3
    g, beta = oracle.gates(a, b, _A_LOG, _DT_BIAS)
    p = np.array([2, 0, 3, 1])
    gp, bp = oracle.gates(a[:, p], b[:, p], _A_LOG[p], _DT_BIAS[p])
    assert np.array_equal(gp, g[:, p]) and np.array_equal(bp, beta[:, p])


def test_l2norm_closed_forms():
    """(3, 4, 0, ...) -> (3, 4, 0, ...) / sqrt(25 + eps); a row 1e-4 e_1 shows where
    eps sits (reading G2, inside the square root): 1e-4 / sqrt(1e-8 + 1e-6),
    not 1e-4 / (1e-4 + 1e-6); a zero row stays zero."""
    x = np.zeros((3, 1, 8))
    x[0, 0, :2] = (3.0, 4.0)
    x[1, 0, 0] = 1e-4
    y = oracle.l2norm(x)
    assert np.allclose(y[0, 0, :2], np.array([3.0, 4.0]) / math.sqrt(25.0 + 1e-6), rtol=1e-15, atol=0)
    assert abs(y[1, 0, 0] - 1e-4 / math.sqrt(1e-8 + 1e-6)) < 1e-16
    assert abs(y[1, 0, 0] - 0.0995037190209989) < 1e-15
    assert np.array_equal(y[2], np.zeros((1, 8)))


def test_l2norm_unit_rows():
    x = gdn_synth.gaussian(33, (10, 3, 64))
    y = oracle.l2norm(x)
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-6)
    # each row keeps its direction: y is a positive multiple of x
    assert np.allclose(y * np.linalg.norm(x.astype(np.float64), axis=-1, keepdims=True), x, rtol=1e-6, atol=0)


# -------------------------------------------------------------------- scan --
def _orthonormal(seed, n, K):
    g = gdn_synth.rng(seed)
    Q, _ = np.linalg.qr(g.standard_normal((K, K)))
    return Q[:, :n].T.copy()


@pytest.mark.parametrize("form", [oracle.FORM_PAGES, oracle.FORM_STANDARD])
def test_delta_rule_overwrite_retrieves_values(form):
    """alpha = beta = 1 with orthonormal keys: each write overwrites the state
    along its key, so S_n^T k_i = v_i and querying with k_i returns
    v_i / sqrt(K) (review page, mechanism step 3, paper sec.5.3)."""
    K = V = 16
    n = 10
    keys = _orthonormal(40, n, K)
    g = gdn_synth.rng(41)
    v = g.standard_normal((1, n, 1, V))
    k = keys.reshape(1, n, 1, K)
    q = keys[::-1].reshape(1, n, 1, K).copy()
    S0 = g.standard_normal((1, 1, K, V))
    zeros = np.zeros((1, n, 1))
    o, S = oracle.scan(q, k, v, zeros, np.ones((1, n, 1)), form=form, S0=S0)
    for i in range(n):
        assert np.allclose(S[0, 0].T @ keys[i], v[0, i, 0], atol=1e-12)
    # the last query is k_0, read after all writes
    assert np.allclose(o[0, n - 1, 0], v[0, 0, 0] / np.sqrt(K), atol=1e-12)


def test_beta_zero_is_pure_decay():
    B, T, Hk, Hv, K, V = 1, 9, 1, 2, 8, 8
    q, k, v, g, beta = gdn_synth.scan_inputs(50, B, T, Hk, Hv, K, V)
    S0 = gdn_synth.gaussian(51, (B, Hv, K, V))
    o, S = oracle.scan(q, k, v, g, np.zeros_like(beta), S0=S0)
    G = np.cumsum(g.astype(np.float64), axis=1)
    for h in range(Hv):
        assert np.allclose(S[0, h], np.exp(G[0, -1, h]) * S0[0, h], rtol=1e-13)
        for t in range(T):
            want = np.exp(G[0, t, h]) * S0[0, h].T @ q[0, t, 0] / np.sqrt(K)
            assert np.allclose(o[0, t, h], want, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("form", [oracle.FORM_PAGES, oracle.FORM_STANDARD])
def test_scan_matches_matrix_product_form(form):
    """PAGES: S_t = (alpha I - beta k k^T) S + beta k v^T; STANDARD (the usual
    Gated DeltaNet form): S_t = alpha (I - beta k k^T) S + beta k v^T; built
    here with numpy matrix products.  GQA: value head h reads key head h*Hk//Hv."""
    B, T, Hk, Hv, K, V = 2, 7, 2, 4, 6, 5
    q, k, v, g, beta = gdn_synth.scan_inputs(60, B, T, Hk, Hv, K, V, alpha_lo=0.5)
    S0 = gdn_synth.gaussian(61, (B, Hv, K, V))
    o, S = oracle.scan(q, k, v, g, beta, form=form, S0=S0, scale=0.37)
    for bb in range(B):
        for h in range(Hv):
            hk = h * Hk // Hv
            St = S0[bb, h].astype(np.float64)
            for t in range(T):
                kt = k[bb, t, hk].astype(np.float64)
                a, bt = math.exp(g[bb, t, h]), float(beta[bb, t, h])
                if form == oracle.FORM_PAGES:
                    St = (a * np.eye(K) - bt * np.outer(kt, kt)) @ St + bt * np.outer(kt, v[bb, t, h])
                else:
                    St = a * (np.eye(K) - bt * np.outer(kt, kt)) @ St + bt * np.outer(kt, v[bb, t, h])
                assert np.allclose(o[bb, t, h], 0.37 * St.T @ q[bb, t, hk], rtol=1e-12, atol=1e-12)
            assert np.allclose(S[bb, h], St, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("form", [oracle.FORM_PAGES, oracle.FORM_STANDARD])
@pytest.mark.parametrize("T,C", [(100, 16), (64, 64), (5, 8), (33, 32)])
def test_chunked_form_equals_recurrence(form, T, C):
    B, Hk, Hv, K, V = 1, 1, 2, 8, 6
    q, k, v, g, beta = gdn_synth.scan_inputs(70 + T, B, T, Hk, Hv, K, V, alpha_lo=0.3)
    S0 = gdn_synth.gaussian(71, (B, Hv, K, V))
    o1, S1 = oracle.scan(q, k, v, g, beta, form=form, S0=S0)
    o2, S2 = oracle.scan_chunked(q, k, v, g, beta, chunk=C, form=form, S0=S0)
    assert np.max(np.abs(o1 - o2)) < 1e-12 * max(1, np.abs(o1).max())
    assert np.max(np.abs(S1 - S2)) < 1e-12 * max(1, np.abs(S1).max())


def test_chunked_handles_underflowing_decay():
    B, T, Hk, Hv, K, V = 1, 40, 1, 1, 8, 4
    q, k, v, g, beta = gdn_synth.scan_inputs(80, B, T, Hk, Hv, K, V)
    g[:] = -400.0       # alpha = e^-400: the cumulative decay underflows double
    o1, S1 = oracle.scan(q, k, v, g, beta)
    o2, S2 = oracle.scan_chunked(q, k, v, g, beta, chunk=16)
    assert np.all(np.isfinite(o2)) and np.allclose(o1, o2, atol=1e-12)


def test_state_chaining_is_exact():
    B, T, Hk, Hv, K, V = 1, 50, 1, 2, 8, 8
    q, k, v, g, beta = gdn_synth.scan_inputs(90, B, T, Hk, Hv, K, V)
    o, S = oracle.scan(q, k, v, g, beta)
    t = 23
    oa, Sa = oracle.scan(q[:, :t], k[:, :t], v[:, :t], g[:, :t], beta[:, :t])
    ob, Sb = oracle.scan(q[:, t:], k[:, t:], v[:, t:], g[:, t:], beta[:, t:], S0=Sa)
    assert np.array_equal(np.concatenate([oa, ob], 1), o) and np.array_equal(Sb, S)


def test_impulse_propagates_linearly():
    """The recurrence is affine in the state: a state impulse D evolves as
    D_t = (alpha_t I - beta_t k k^T) D_{t-1} (PAGES form), whatever v is
    (review page, mechanism step 3, impulse study, Fig.1b)."""
    B, T, Hk, Hv, K, V = 1, 30, 1, 1, 8, 8
    q, k, v, g, beta = gdn_synth.scan_inputs(95, B, T, Hk, Hv, K, V, alpha_lo=0.8)
    S0 = gdn_synth.gaussian(96, (B, Hv, K, V))
    D0 = gdn_synth.gaussian(97, (B, Hv, K, V), std=0.01)
    _, Sa = oracle.scan(q, k, v, g, beta, S0=S0)
    _, Sb = oracle.scan(q, k, v, g, beta, S0=S0.astype(np.float64) + D0.astype(np.float64))
    D = D0[0, 0].astype(np.float64)
    for t in range(T):
        kt = k[0, t, 0].astype(np.float64)
        D = (math.exp(g[0, t, 0]) * np.eye(K) - beta[0, t, 0] * np.outer(kt, kt)) @ D
    assert np.allclose(Sb[0, 0] - Sa[0, 0], D, atol=1e-13)


def test_layer_oracle_composes_on_tiny_shapes():
    sh = gdn_synth.TINY
    _, x = gdn_synth.activations(0, 64, sh.H, hot="fixed")
    W_in = gdn_synth.weights(100, sh.n_in, sh.H)
    W_out = gdn_synth.weights(101, sh.H, sh.Hv * sh.V)
    A_log, dt_bias = gdn_synth.gate_params(102, sh.Hv)
    st = oracle.layer_forward(x, oracle.quantize(W_in), oracle.quantize(W_out), A_log, dt_bias,
                              1, 64, sh.Hk, sh.Hv, sh.K, sh.V, stages=True)
    assert st["P"].shape == (64, sh.n_in) and st["y"].shape == (64, sh.H)
    assert np.all(np.isfinite(st["y"]))
    # the W4A4 layer output sits near the float64 unquantised layer output (A4/W4 noise level)
    P = x.astype(np.float64) @ W_in.astype(np.float64).T
    q, k, v, _z, a, b = oracle.split_projection(P, sh.Hk, sh.Hv, sh.K, sh.V)
    g, beta = oracle.gates(a, b, A_log, dt_bias)
    o, _ = oracle.scan(oracle.l2norm(q.reshape(1, 64, sh.Hk, sh.K)), oracle.l2norm(k.reshape(1, 64, sh.Hk, sh.K)),
                       v.reshape(1, 64, sh.Hv, sh.V), g.reshape(1, 64, sh.Hv), beta.reshape(1, 64, sh.Hv))
    y = o.reshape(64, -1) @ W_out.astype(np.float64).T
    rel = np.linalg.norm(st["y"] - y) / np.linalg.norm(y)
    assert rel < 0.5


# ------------------------------------------------------------- output gate --
# Reading O1 (the pages name the z projection as one that moves y and keep the
# norms unquantised, but give no formula): G = RMSNorm(o) * w * SiLU(z) per token
# and value head.  Pinned by closed forms and invariants, not by its formula.
def test_output_gate_silu_closed_forms():
    """o = ones (RMS 1, eps 0), w = 1: G = SiLU(z); sigmoid(+-ln 3) = 3/4, 1/4."""
    ln3 = np.log(3.0)
    z = np.array([[[ln3, -ln3, 0.0, 60.0]]])
    G = oracle.output_gate(np.ones((1, 1, 4)), z, np.ones(4), eps=0.0)
    np.testing.assert_allclose(G[0, 0], [0.75 * ln3, -0.25 * ln3, 0.0, 60.0], rtol=1e-15, atol=1e-15)


def test_output_gate_normalises_by_the_mean_square():
    """One-hot o over V = 4 channels: mean square 1/4, so the normalised row is 2 e_1;
    with z = 60 (SiLU(z) = z to double precision) and w = 1/z the gate output is
    that row, and any row's output has mean square 1."""
    z = np.full((1, 1, 4), 60.0)
    w = np.full(4, 1.0 / 60.0)
    G = oracle.output_gate(np.array([[[0.0, 1.0, 0.0, 0.0]]]), z, w, eps=0.0)
    np.testing.assert_allclose(G[0, 0], [0.0, 2.0, 0.0, 0.0], rtol=1e-14, atol=1e-15)
    o = gdn_synth.gaussian(7, (3, 2, 4), std=5.0)
    G = oracle.output_gate(o, np.full(o.shape, 60.0), w, eps=0.0)
    np.testing.assert_allclose((G ** 2).mean(axis=-1), 1.0, rtol=1e-13)


def test_output_gate_scale_invariance_and_zero_gate():
    """RMSNorm ignores a positive scale of o (eps 0); z = 0 closes the gate; the
    per-channel weight multiplies channel i of every head."""
    o = gdn_synth.gaussian(8, (5, 3, 8), std=1.0).astype(np.float64)
    z = gdn_synth.gaussian(9, (5, 3, 8), std=2.0).astype(np.float64)
    w = gdn_synth.gaussian(10, (8,), std=1.0).astype(np.float64)
    G = oracle.output_gate(o, z, w, eps=0.0)
    np.testing.assert_allclose(oracle.output_gate(3.7 * o, z, w, eps=0.0), G, rtol=1e-13, atol=1e-14)
    assert np.all(oracle.output_gate(o, np.zeros_like(z), w) == 0.0)
    G1 = oracle.output_gate(o, z, np.ones(8), eps=0.0)
    np.testing.assert_allclose(G, G1 * w, rtol=1e-13, atol=1e-14)
    # a zero row stays zero (eps keeps it finite)
    o[2, 1] = 0.0
    assert np.all(oracle.output_gate(o, z, w)[2, 1] == 0.0)


def test_layer_oracle_gate_option_routes_z():
    """With the gate, the layer's out_proj input is G computed from the scan output
    and the projection's z slice; a gate weight of zero gives y = 0."""
    sh = gdn_synth.TINY
    _, x = gdn_synth.activations(1, 64, sh.H, hot="fixed")
    W_in = oracle.quantize(gdn_synth.weights(110, sh.n_in, sh.H))
    W_out = oracle.quantize(gdn_synth.weights(111, sh.H, sh.Hv * sh.V))
    A_log, dt_bias = gdn_synth.gate_params(112, sh.Hv)
    w = gdn_synth.gaussian(113, (sh.V,), std=1.0)
    st = oracle.layer_forward(x, W_in, W_out, A_log, dt_bias, 1, 64, sh.Hk, sh.Hv, sh.K, sh.V, stages=True,
                              out_norm=w)
    z = oracle.split_projection(st["P"], sh.Hk, sh.Hv, sh.K, sh.V)[3]
    o32 = st["o"].reshape(64, sh.Hv, sh.V).astype(np.float32)
    np.testing.assert_allclose(st["G"], oracle.output_gate(o32, z.reshape(64, sh.Hv, sh.V), w), rtol=0, atol=0)
    y0 = oracle.layer_forward(x, W_in, W_out, A_log, dt_bias, 1, 64, sh.Hk, sh.Hv, sh.K, sh.V,
                              out_norm=np.zeros(sh.V))[0]
    assert np.all(y0 == 0.0)


# -------------------------------------------------------- short convolution --
# Reading C1 (the pages keep convolutions unquantised and say nothing else): a
# causal depthwise convolution of width W on the q|k|v channels, then SiLU.
def test_short_conv_matches_numpy_convolve():
    """Pre-activation per channel = the first T terms of numpy.convolve with the
    reversed taps (zero history)."""
    B, T, C, W = 2, 11, 5, 4
    x = gdn_synth.gaussian(30, (B * T, C), std=1.0).astype(np.float64)
    w = gdn_synth.gaussian(31, (C, W), std=1.0).astype(np.float64)
    out = oracle.short_conv(x, w, B, T, silu=False)
    for b in range(B):
        for c in range(C):
            ref = np.convolve(x[b * T:(b + 1) * T, c], w[c, ::-1])[:T]
            np.testing.assert_allclose(out[b * T:(b + 1) * T, c], ref, rtol=1e-14, atol=1e-14)


def test_short_conv_taps_and_silu_closed_form():
    """The last tap alone gives SiLU(x_t) (SiLU(ln 3) = 0.75 ln 3); the first tap
    alone gives SiLU(x_{t-3}), zero for the first three tokens."""
    ln3 = np.log(3.0)
    x = np.full((6, 1), ln3)
    out = oracle.short_conv(x, np.array([[0.0, 0.0, 0.0, 1.0]]), 1, 6)
    np.testing.assert_allclose(out[:, 0], 0.75 * ln3, rtol=1e-15)
    x = np.arange(1, 7, dtype=np.float64).reshape(6, 1)
    out = oracle.short_conv(x, np.array([[1.0, 0.0, 0.0, 0.0]]), 1, 6, silu=False)
    np.testing.assert_array_equal(out[:, 0], [0.0, 0.0, 0.0, 1.0, 2.0, 3.0])


def test_short_conv_is_causal_and_chains():
    """Changing token 7 leaves tokens 0..6 alone; convolving T1 then T2 tokens with
    the carried state equals convolving T1 + T2 at once (T2 shorter than the
    window included), and the state holds the last W-1 inputs."""
    T, C, W = 16, 6, 4
    x = gdn_synth.gaussian(32, (T, C), std=1.0).astype(np.float64)
    w = gdn_synth.gaussian(33, (C, W), std=1.0).astype(np.float64)
    full, st_full = oracle.short_conv(x, w, 1, T, return_state=True)
    x2 = x.copy()
    x2[7] += 5.0
    out2 = oracle.short_conv(x2, w, 1, T)
    np.testing.assert_array_equal(out2[:7], full[:7])
    assert np.all(out2[7] != full[7])
    for t1 in (1, 2, 9, 15):
        a, st = oracle.short_conv(x[:t1], w, 1, t1, return_state=True)
        b, st2 = oracle.short_conv(x[t1:], w, 1, T - t1, state_in=st, return_state=True)
        np.testing.assert_array_equal(np.concatenate([a, b]), full)
        np.testing.assert_array_equal(st2, st_full)
    np.testing.assert_array_equal(st_full[0], x[T - (W - 1):].T)


def test_layer_oracle_conv_option():
    """The convolution feeds q|k|v only: z, a, b and the gates see the raw projection;
    an identity-tap convolution equals applying SiLU to q|k|v."""
    sh = gdn_synth.TINY
    _, x = gdn_synth.activations(2, 32, sh.H, hot="fixed")
    W_in = oracle.quantize(gdn_synth.weights(120, sh.n_in, sh.H))
    W_out = oracle.quantize(gdn_synth.weights(121, sh.H, sh.Hv * sh.V))
    A_log, dt_bias = gdn_synth.gate_params(122, sh.Hv)
    C = 2 * sh.Hk * sh.K + sh.Hv * sh.V
    taps = np.zeros((C, 4))
    taps[:, 3] = 1.0
    st = oracle.layer_forward(x, W_in, W_out, A_log, dt_bias, 1, 32, sh.Hk, sh.Hv, sh.K, sh.V, stages=True,
                              conv_w=taps)
    P = st["P"]
    np.testing.assert_allclose(st["Pc"][:, :C], P[:, :C] / (1.0 + np.exp(-P[:, :C])), rtol=1e-15)
    np.testing.assert_array_equal(st["Pc"][:, C:], P[:, C:])


# ------------------------------------------------------ state passing (P1) --
@pytest.mark.parametrize("form", [oracle.FORM_PAGES, oracle.FORM_STANDARD])
def test_transition_of_one_token_is_the_closed_form(form):
    """One token: P = a I - b k k^T (PAGES) or a (I - b k k^T) (STANDARD), and
    the query map is scale P^T q (Eq.(2) written as a map of the state)."""
    B, T, Hk, Hv, K = 1, 1, 1, 2, 6
    q, k, _, g, beta = gdn_synth.scan_inputs(200, B, T, Hk, Hv, K, 4, alpha_lo=0.5)
    P, m = oracle.scan_transition(q, k, g, beta, scale=0.3, form=form)
    kt = k[0, 0, 0].astype(np.float64)
    for h in range(Hv):
        a, bt = math.exp(g[0, 0, h]), float(beta[0, 0, h])
        want = (a * np.eye(K) - bt * np.outer(kt, kt)) if form == oracle.FORM_PAGES else \
            a * (np.eye(K) - bt * np.outer(kt, kt))
        assert np.allclose(P[0, h], want, rtol=0, atol=1e-15)
        assert np.allclose(m[0, 0, h], 0.3 * want.T @ q[0, 0, 0], rtol=0, atol=1e-15)


def test_transition_without_writes_is_the_decay():
    """beta = 0: nothing is written, the state only decays, so P_t is the
    running product of the alphas times I and m_t = scale (prod alpha) q_t."""
    B, T, Hk, Hv, K = 1, 9, 1, 1, 5
    q, k, _, g, beta = gdn_synth.scan_inputs(201, B, T, Hk, Hv, K, 4, alpha_lo=0.6)
    beta[:] = 0.0
    P, m = oracle.scan_transition(q, k, g, beta, scale=1.0)
    run = np.cumprod(np.exp(g[0, :, 0].astype(np.float64)))
    assert np.allclose(P[0, 0], run[-1] * np.eye(K), rtol=1e-14, atol=0)
    for t in range(T):
        assert np.allclose(m[0, t, 0], run[t] * q[0, t, 0], rtol=1e-14, atol=1e-16)


def test_transition_full_overwrite_is_a_projector():
    """alpha = 1, beta = 1, unit k: each token erases the state along k
    (review page, sec.5.3, the overwrite along the key direction), so the map
    of a token is the projector I - k k^T; repeating the same key changes
    nothing, and two orthogonal keys erase both directions."""
    B, T, Hk, Hv, K = 1, 3, 1, 1, 6
    q, k, _, g, beta = gdn_synth.scan_inputs(202, B, T, Hk, Hv, K, 4)
    g[:] = 0.0
    beta[:] = 1.0
    k[0, :, 0] = k[0, 0, 0]
    P, _ = oracle.scan_transition(q, k, g, beta)
    k0 = k[0, 0, 0].astype(np.float64)
    proj = np.eye(K) - np.outer(k0, k0)
    assert np.allclose(P[0, 0], proj, atol=1e-15) and np.allclose(P[0, 0] @ P[0, 0], P[0, 0], atol=1e-15)
    e = np.eye(K)
    k2 = np.zeros((B, 2, Hk, K), np.float32)
    k2[0, 0, 0], k2[0, 1, 0] = e[1], e[4]
    P2, _ = oracle.scan_transition(q[:, :2], k2, g[:, :2], beta[:, :2])
    want = np.eye(K)
    want[1, 1] = want[4, 4] = 0.0
    assert np.array_equal(P2[0, 0], want)


@pytest.mark.parametrize("form", [oracle.FORM_PAGES, oracle.FORM_STANDARD])
@pytest.mark.parametrize("bounds", [[0, 50], [0, 1, 50], [0, 17, 18, 40, 50], [0, 25, 50]])
def test_segmented_scan_equals_the_recurrence(form, bounds):
    """Spans scanned from zero, joined through their maps, give the recurrence
    over the whole sequence (outputs and final state), with a random start."""
    B, T, Hk, Hv, K, V = 2, 50, 2, 4, 8, 6
    q, k, v, g, beta = gdn_synth.scan_inputs(203, B, T, Hk, Hv, K, V, alpha_lo=0.7)
    S0 = gdn_synth.gaussian(204, (B, Hv, K, V))
    o1, S1 = oracle.scan(q, k, v, g, beta, form=form, S0=S0)
    o2, S2 = oracle.scan_segmented(q, k, v, g, beta, bounds, form=form, S0=S0)
    assert np.max(np.abs(o1 - o2)) < 1e-12 * max(1, np.abs(o1).max())
    assert np.max(np.abs(S1 - S2)) < 1e-12 * max(1, np.abs(S1).max())


def test_state_combine_and_correction_by_hand():
    """The two joining steps written out with explicit loops on a tiny case."""
    r = np.random.default_rng(205)
    P, S_loc, S_in = r.standard_normal((2, 3, 3)), r.standard_normal((2, 3, 2)), r.standard_normal((2, 3, 2))
    got = oracle.state_combine(P, S_loc, S_in)
    for n in range(2):
        for i in range(3):
            for j in range(2):
                assert math.isclose(got[n, i, j], sum(P[n, i, l] * S_in[n, l, j] for l in range(3)) + S_loc[n, i, j],
                                    rel_tol=1e-14, abs_tol=1e-14)
    o_loc, m = r.standard_normal((1, 2, 2, 2)), r.standard_normal((1, 2, 2, 3))
    S = r.standard_normal((1, 2, 3, 2))
    got = oracle.output_correct(o_loc, m, S)
    for t in range(2):
        for h in range(2):
            for j in range(2):
                want = o_loc[0, t, h, j] + sum(S[0, h, i, j] * m[0, t, h, i] for i in range(3))
                assert math.isclose(got[0, t, h, j], want, rel_tol=1e-14, abs_tol=1e-14)
