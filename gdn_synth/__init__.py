"""Seeded synthetic inputs shared by the CUDA-path tests, the benchmark and the
oracle.  This module draws random numbers and nothing else: it holds none of
the layer's arithmetic (no quantisation, no gates, no recurrence).

Distributions follow the workloads the review page of "Why Gated DeltaNet
Survives 4-Bit Quantization" describes for the residual stream (paper
sec.5.1, Table 2: heavy-tailed activations with a few hot channels ~100x the
median): N(0,1) activations with a small set of channels scaled 50-100x,
N(0, 0.02) weights, A_log ~ U(log 1, log 16), dt_bias ~ N(0, 0.5).

bf16 activations are returned as raw uint16 bit patterns plus the same values
widened to float32 (exact); the float32 -> bf16 rounding here is plain
round-to-nearest-even on the bit pattern, a property of the input, not of the
method.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class LayerShape:
    H: int        # hidden size
    Hk: int       # key heads
    Hv: int       # value heads
    K: int        # key head dim
    V: int        # value head dim

    @property
    def n_in(self) -> int:
        """Fused in_proj width q | k | v | z | a | b."""
        return 2 * self.Hk * self.K + 2 * self.Hv * self.V + 2 * self.Hv

    @property
    def slices(self):
        return [("q", self.Hk * self.K), ("k", self.Hk * self.K), ("v", self.Hv * self.V),
                ("z", self.Hv * self.V), ("a", self.Hv), ("b", self.Hv)]


TINY = LayerShape(H=256, Hk=2, Hv=2, K=64, V=64)
FULL = LayerShape(H=5120, Hk=16, Hv=32, K=128, V=128)


def activations(seed: int, rows: int, cols: int, hot: str = "percent", hot_n: int = 2,
                hot_frac: float = 0.01, lo: float = 50.0, hi: float = 100.0, dtype=np.float32):
    """N(0,1) activations with hot channels.

    hot="fixed": ``hot_n`` seeded channels scaled x100.
    hot="percent": ``hot_frac`` of the channels scaled U(lo, hi).
    hot="none": plain N(0,1).
    Returns (bf16 bits [rows, cols], float32 values of those bits)."""
    g = rng(seed)
    x = g.standard_normal((rows, cols), dtype=np.float32)
    if hot == "fixed":
        ch = g.choice(cols, size=hot_n, replace=False)
        x[:, ch] *= 100.0
    elif hot == "percent":
        n = max(1, int(round(hot_frac * cols)))
        ch = g.choice(cols, size=n, replace=False)
        x[:, ch] *= g.uniform(lo, hi, size=n).astype(np.float32)
    bits = to_bf16_bits(x)
    return bits, bf16_bits_to_f32(bits)


def weights(seed: int, rows: int, cols: int, std: float = 0.02, slice_rows=None, slice_gain=None):
    """N(0, std) float32 weights [rows, cols]; optional per-slice gains (rows
    partitioned by ``slice_rows``) so per-module amax differ."""
    g = rng(seed)
    w = g.standard_normal((rows, cols), dtype=np.float32) * np.float32(std)
    if slice_rows is not None:
        r0 = 0
        for n, gain in zip(slice_rows, slice_gain):
            w[r0:r0 + n] *= np.float32(gain)
            r0 += n
    return w


def gate_params(seed: int, Hv: int, alog_lo: float = 0.0, alog_hi: float = math.log(16.0)):
    g = rng(seed)
    A_log = g.uniform(alog_lo, alog_hi, size=Hv).astype(np.float32)
    dt_bias = (g.standard_normal(Hv) * 0.5).astype(np.float32)
    return A_log, dt_bias


def scan_inputs(seed: int, B: int, T: int, Hk: int, Hv: int, K: int, V: int,
                alpha_lo: float = 0.9, alpha_hi: float = 0.9999, beta_lo: float = 0.0,
                beta_hi: float = 1.0, normalise: bool = True):
    """Direct inputs for the recurrence: unit-norm q, k (when ``normalise``;
    the normalisation here is input preparation, drawn directions), N(0,1) v,
    log-decay g = log U(alpha_lo, alpha_hi), beta ~ U(beta_lo, beta_hi).
    All float32."""
    gg = rng(seed)
    q = gg.standard_normal((B, T, Hk, K), dtype=np.float32)
    k = gg.standard_normal((B, T, Hk, K), dtype=np.float32)
    if normalise:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = gg.standard_normal((B, T, Hv, V), dtype=np.float32)
    g = np.log(gg.uniform(alpha_lo, alpha_hi, size=(B, T, Hv))).astype(np.float32)
    beta = gg.uniform(beta_lo, beta_hi, size=(B, T, Hv)).astype(np.float32)
    return q, k, v, g, beta


def gaussian(seed: int, shape, std: float = 1.0, dtype=np.float32):
    return (rng(seed).standard_normal(shape) * std).astype(dtype)


# ------------------------------------------------------------ named workloads
GEMM_SLICES = (2048, 2048, 4096, 4096)
GEMM_SLICE_GAIN = (1.0, 2.0, 4.0, 1.0)

WORKLOADS = {
    "tiny_layer": dict(shape=TINY, B=1, T=64, seed=0, hot="fixed"),
    "gemm_8192x12288x5120": dict(M=8192, N=12288, K=5120, seed=1),
    "prefill_T4096": dict(shape=FULL, B=1, T=4096, seed=2, hot="percent"),
    "prefill_T32768": dict(shape=FULL, B=1, T=32768, seed=3, hot="percent", impulse_t=1000),
    "decode_B64": dict(shape=FULL, B=64, steps=256, prefill_T=1024, seed=4),
}
