"""GPU NVFP4 quantiser vs the oracle: packed E2M1 codes, E4M3 scales (atom
layout) and the global scale must be bit-exact."""
import numpy as np
import pytest
import torch

import gdn_synth
import nvfp4_w4a4_gated_b200 as nv
import oracle
from gpu_util import bf16_device, f32_device

pytestmark = pytest.mark.gpu


def _check(x_dev, x_f32, S=None):
    rows, cols = x_f32.shape
    if S is None:
        q = nv.nvfp4_quantize(x_dev)
        ref = oracle.quantize(x_f32)
    else:
        out = nv.NVFP4Matrix.empty(rows, cols)
        out.scale.fill_(float(S))
        q = nv.nvfp4_quantize(x_dev, out=out, given_scale=True)
        ref = oracle.quantize(x_f32, S=S)
    torch.cuda.synchronize()
    nv.check_device_error()
    codes, sf, S_ref = ref
    assert q.scale.item() == float(S_ref)
    got_codes = q.codes.cpu().numpy()
    bad = np.argwhere(got_codes != codes)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:5].tolist()}"
    assert np.array_equal(q.sf.cpu().numpy(), oracle.sf_linear_to_mma(sf, rows, cols))


@pytest.mark.parametrize("rows,cols,hot", [(1, 64, "none"), (64, 256, "fixed"), (100, 128, "percent"),
                                           (300, 512, "percent"), (129, 320, "fixed"), (1000, 5120, "percent")])
def test_quantize_bf16_matches_oracle(cuda_dev, rows, cols, hot):
    bits, x = gdn_synth.activations(rows * 7 + cols, rows, cols, hot=hot)
    _check(bf16_device(bits), x)


@pytest.mark.parametrize("rows,cols", [(64, 128), (257, 384), (2048, 4096)])
def test_quantize_fp32_matches_oracle(cuda_dev, rows, cols):
    g = gdn_synth.rng(rows + cols)
    # wide dynamic range, exact zeros, negative values and near-tie magnitudes
    x = (g.standard_normal((rows, cols)) * np.exp(g.uniform(-12, 6, (rows, cols)))).astype(np.float32)
    x[::7, ::5] = 0.0
    x[3, :16] = 0.0
    _check(f32_device(x), x)


def test_quantize_given_scale_harmonised_slices(cuda_dev):
    sl, gain = (64, 64, 128), (1.0, 4.0, 2.0)
    W = gdn_synth.weights(5, sum(sl), 256, slice_rows=sl, slice_gain=gain)
    S = oracle.global_scale(W)
    r0 = 0
    for n in sl:
        _check(f32_device(W[r0:r0 + n]), W[r0:r0 + n], S=S)
        r0 += n
    _check(f32_device(W), W)


def test_quantize_zero_and_strided(cuda_dev):
    x = np.zeros((130, 64), np.float32)
    _check(f32_device(x), x)
    bits, xf = gdn_synth.activations(9, 70, 384, hot="fixed")
    big = torch.zeros((70, 512), dtype=torch.bfloat16, device="cuda")
    big[:, :384] = bf16_device(bits)
    q = nv.nvfp4_quantize(big[:, :384])
    codes, sf, S = oracle.quantize(xf)
    assert q.scale.item() == float(S)
    assert np.array_equal(q.codes.cpu().numpy(), codes)
    assert np.array_equal(q.sf.cpu().numpy(), oracle.sf_linear_to_mma(sf, 70, 384))


def test_quantize_full_size_activation(cuda_dev):
    """The 8192 x 5120 outlier-heavy activation of the standalone GEMM workload, every byte."""
    bits, x = gdn_synth.activations(1, 8192, 5120, hot="percent")
    _check(bf16_device(bits), x)


def test_quantize_full_size_weight(cuda_dev):
    """The fused in_proj weight [12352 x 5120] quantised as one tensor (harmonised scale)."""
    sh = gdn_synth.FULL
    W = gdn_synth.weights(200, sh.n_in, sh.H)
    _check(f32_device(W), W)


@pytest.mark.parametrize("amax", [2688.0, 1000.0, 3.3e-3, 7.77e5])
def test_quantize_block_maxima_near_e4m3_midpoints(cuda_dev, amax):
    """Blocks whose max m puts the quotient m / (6 S) within three fp32 ulps of
    every rounding midpoint between consecutive E4M3 values, under four global
    scales: the block scale bytes (and codes) must match the oracle's correctly
    rounded division followed by E4M3 rounding."""
    vals = sorted({oracle.e4m3_decode(b) for b in range(0x7F)})
    S = np.float32(np.float32(amax) / np.float32(2688.0))
    d6 = np.float32(np.float32(6.0) * S)
    maxima = []
    for lo, hi in zip(vals[:-1], vals[1:]):
        m0 = np.float32(np.float32((lo + hi) / 2) * d6)
        for k in range(-3, 4):
            m = m0
            for _ in range(abs(k)):
                m = np.nextafter(m, np.float32(np.inf if k > 0 else 0), dtype=np.float32)
            if 0 < m <= amax:
                maxima.append(m)
    blocks = np.zeros((len(maxima) + 1, 16), np.float32)
    g = gdn_synth.rng(17)
    for i, m in enumerate(maxima):
        blocks[i, 1:] = (g.uniform(-1, 1, 15) * m).astype(np.float32)
        blocks[i, 0] = -m if i % 2 else m
    blocks[-1, 5] = np.float32(amax)
    nblk = (blocks.shape[0] + 3) // 4 * 4
    x = np.zeros((nblk, 16), np.float32)
    x[:blocks.shape[0]] = blocks
    x = x.reshape(-1, 64)
    _check(f32_device(x), x)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rows_split_across_ranks_share_the_tensor_scale(cuda_dev, dtype):
    """A tensor whose rows are split over three (emulated) ranks: each part's
    amax word (AMAX_ONLY), the max over the parts (what a max all-reduce
    gives), then each part quantised from that word (FROM_AMAX).  Every part's
    codes, scales and S must equal the oracle's quantisation of the whole
    tensor restricted to the part's rows."""
    rows, cols = 700, 512
    bits, x = gdn_synth.activations(77, rows, cols, hot="percent")
    dev = bf16_device(bits) if dtype == "bf16" else f32_device(x)
    codes, sf, S = oracle.quantize(x)
    bounds = [0, 129, 130, rows]          # parts of 129, 1 and 570 rows
    words = []
    for a, b in zip(bounds, bounds[1:]):
        ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        nv.nvfp4_quantize(dev[a:b], workspace=ws, mode=nv.QUANT_AMAX_ONLY)
        words.append(ws)
    torch.cuda.synchronize()
    local = [w[:4].view(torch.int32).item() for w in words]
    for (a, b), lw in zip(zip(bounds, bounds[1:]), local):
        assert np.int32(lw).view(np.float32) == np.abs(x[a:b]).max()
    glob = torch.stack([w[:4].view(torch.int32) for w in words]).amax(dim=0)
    for (a, b), ws in zip(zip(bounds, bounds[1:]), words):
        ws[:4].view(torch.int32).copy_(glob)
        q = nv.nvfp4_quantize(dev[a:b], workspace=ws, mode=nv.QUANT_FROM_AMAX)
        torch.cuda.synchronize()
        nv.check_device_error()
        assert q.scale.item() == float(S)
        assert np.array_equal(q.codes.cpu().numpy(), codes[a:b])
        assert np.array_equal(q.sf.cpu().numpy(), oracle.sf_linear_to_mma(sf[a:b], b - a, cols))
