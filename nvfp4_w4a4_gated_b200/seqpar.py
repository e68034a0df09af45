"""Sequence-parallel delta-rule scan: each rank holds one span of every
sequence, and the spans are joined through the recurrence's state.

Eq.(2) of the review page "Why Gated DeltaNet Survives 4-Bit Quantization"
(background) is affine in the state, so a span started from S_in ends in
P S_in + S_loc and its outputs are o_loc + S_in^T m (P, m: the span's maps;
o_loc, S_loc: its zero-start scan).  Per rank:

1. scan the local span from a zero state (o_loc, S_loc) and form its maps
   (P, m): two independent launches on the local tokens;
2. all-gather (P, S_loc): the one exchange, B x Hv x K x (K + V) floats per
   rank, whatever the span length;
3. compose the maps of the ranks before this one, in rank order, starting from
   the sequence's initial state: this rank's S_in;
4. correct the outputs, o = o_loc + S_in^T m, and form the state at the end of
   the span, P S_in + S_loc (the last rank's is the sequence's final state).

The compute steps are the library's kernels (``gdn_scan_span`` for step 1,
``gdn_state_combine`` for step 3 in one launch, ``gdn_scan_correct``);
torch.distributed carries the exchange.  ``ops`` lets the host logic run
against another implementation of the steps (the multi-rank CPU tests use
it); the default is the CUDA library and nothing else.

``sequence_parallel_layer`` composes the whole layer forward around the split
scan.  The pages' NVFP4 format has one FP32 scale per tensor (review page,
background / paper sec.1), so each quantised activation (x, and o before
out_proj) takes its scale from the amax of the whole sequence: every rank
writes the amax of its rows, a max all-reduce joins them, and every rank
quantises its rows from the joined word, so its codes and block scales are
the whole tensor's rows.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import (FORM_PAGES, QUANT_AMAX_ONLY, QUANT_FROM_AMAX, SCAN_AUTO, GdnDims, LayerWeights, gdn_gates,
               gdn_scan_correct, gdn_scan_span, gdn_state_combine, lib, nvfp4_quantize, w4a4_gemm)


class CudaSpanOps:
    """The steps on the GPU, through the C-ABI library."""

    def __init__(self, algo: int = SCAN_AUTO, stream=None):
        self.algo, self.stream = algo, stream

    def local(self, q_hat, k_hat, v, g, beta, B, T, dims, scale, form):
        """Zero-start scan and span maps, one chunk preparation (gdn_scan_span)."""
        return gdn_scan_span(q_hat, k_hat, v, g, beta, B, T, dims, scale=scale, form=form, algo=self.algo,
                             stream=self.stream)

    def combine(self, P, S_loc, S_in):
        """P [m, B, Hv, K, K], S_loc [m, B, Hv, K, V]: the m maps in order, one launch."""
        return gdn_state_combine(P, S_loc, S_in, stream=self.stream)

    def correct(self, qmap, S_in, o, B, T):
        return gdn_scan_correct(qmap, S_in, o, B, T, stream=self.stream)


@dataclass
class SpanLocal:
    """Step 1's results for one span."""
    o: torch.Tensor        # [B*T, Hv, V], zero-start outputs (corrected in place by join)
    S_loc: torch.Tensor    # [B, Hv, K, V]
    P: torch.Tensor        # [B, Hv, K, K]
    qmap: torch.Tensor     # [B*T, Hv, K]


def span_local(q_hat, k_hat, v, g, beta, B: int, T: int, dims: GdnDims, scale: float | None = None,
               form: int = FORM_PAGES, ops=None) -> SpanLocal:
    """Step 1: the span's zero-start scan and its maps."""
    ops = ops or CudaSpanOps()
    return SpanLocal(*ops.local(q_hat, k_hat, v, g, beta, B, T, dims, scale, form))


def span_join(local: SpanLocal, P_before, S_loc_before, B: int, T: int, state_in=None, ops=None):
    """Steps 3 and 4 for one span, given the maps of the spans before it in
    order, stacked (P_before [m, B, Hv, K, K], S_loc_before [m, B, Hv, K, V];
    None or m = 0 when it is the first span), and the sequence's initial state
    (None = zero).  Returns (o, state at the end of the span)."""
    ops = ops or CudaSpanOps()
    S_in = state_in
    if P_before is not None and len(P_before):
        S_in = ops.combine(P_before, S_loc_before, S_in)
    o = local.o
    if S_in is not None:
        o = ops.correct(local.qmap, S_in, o, B, T)
    return o, ops.combine(local.P[None], local.S_loc[None], S_in)


def sequence_parallel_scan(q_hat, k_hat, v, g, beta, B: int, T: int, dims: GdnDims, scale: float | None = None,
                           form: int = FORM_PAGES, state_in=None, group=None, ops=None):
    """The delta-rule scan of B sequences whose tokens are split across the
    ranks of ``group`` in rank order: this rank holds T consecutive tokens of
    every sequence (q_hat, k_hat [B*T, Hk, K]; v [B*T, >=Hv*V]; g, beta
    [B*T, Hv]), and every rank passes the same ``state_in`` (the sequences'
    initial state, or None).  Returns (o [B*T, Hv, V] for the local tokens, the
    state after the local span [B, Hv, K, V]).  Every rank must call it with
    the same B and dims; span lengths may differ."""
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    local = span_local(q_hat, k_hat, v, g, beta, B, T, dims, scale, form, ops)
    if world == 1:
        return span_join(local, None, None, B, T, state_in, ops)
    P_all = torch.empty((world,) + tuple(local.P.shape), dtype=local.P.dtype, device=local.P.device)
    S_all = torch.empty((world,) + tuple(local.S_loc.shape), dtype=local.S_loc.dtype, device=local.S_loc.device)
    dist.all_gather(list(P_all.unbind(0)), local.P.contiguous(), group=group)
    dist.all_gather(list(S_all.unbind(0)), local.S_loc.contiguous(), group=group)
    return span_join(local, P_all[:rank], S_all[:rank], B, T, state_in, ops)


def segmented_scan(spans, B: int, dims: GdnDims, scale: float | None = None, form: int = FORM_PAGES,
                   state_in=None, ops=None):
    """The same algorithm on one device, with the spans of every sequence given
    as a list of (q_hat, k_hat, v, g, beta, T) tuples in order: all spans'
    step 1 first (independent), then the joins in order, each span starting
    from the state the previous join produced.  Returns the list of span
    outputs and the final state."""
    locals_ = [span_local(q, k, v, g, b, B, T, dims, scale, form, ops) for (q, k, v, g, b, T) in spans]
    outs, S = [], state_in
    for loc, span in zip(locals_, spans):
        o, S = span_join(loc, None, None, B, span[5], S, ops)
        outs.append(o)
    return outs, S


# ------------------------------------------------------------ the layer --
class CudaLayerOps(CudaSpanOps):
    """The layer's steps on the GPU, through the C-ABI library."""

    def amax_word(self, x):
        """int32 [1] holding the float bits of max|x| (workspace word 0 of an
        NVFP4_QUANT_AMAX_ONLY quantisation)."""
        ws = torch.zeros(max(16, lib().nvfp4_quantize_workspace_size()), dtype=torch.uint8, device=x.device)
        nvfp4_quantize(x, workspace=ws, stream=self.stream, mode=QUANT_AMAX_ONLY)
        return ws[:4].view(torch.int32)

    def quantize_from_amax(self, x, word):
        ws = torch.zeros(max(16, lib().nvfp4_quantize_workspace_size()), dtype=torch.uint8, device=x.device)
        ws[:4].view(torch.int32).copy_(word)
        return nvfp4_quantize(x, workspace=ws, stream=self.stream, mode=QUANT_FROM_AMAX)

    def gemm(self, a, b):
        return w4a4_gemm(a, b, stream=self.stream)

    def gates(self, P, w: LayerWeights):
        """(q_hat, k_hat, v, g, beta) of the fused projection's rows."""
        d = w.dims
        q_hat, k_hat, g, beta = gdn_gates(P, d, w.A_log, w.dt_bias, stream=self.stream)
        c0 = 2 * d.Hk * d.K
        return q_hat, k_hat, P[:, c0:c0 + d.Hv * d.V], g, beta


def _quantize_across(x, ops, group, distributed):
    """x quantised with the scale of the whole tensor split across the ranks."""
    word = ops.amax_word(x)
    if distributed:
        dist.all_reduce(word, op=dist.ReduceOp.MAX, group=group)   # non-negative floats order as their bits
    return ops.quantize_from_amax(x, word)


def sequence_parallel_layer(w, x, B: int, T: int, form: int = FORM_PAGES, state_in=None, group=None, ops=None):
    """One GDN layer forward under NVFP4 W4A4 for B sequences whose tokens are
    split across the ranks of ``group`` in rank order: this rank holds T
    consecutive tokens of every sequence (x [B*T, hidden], rows (b, t)).  The
    steps are the layer's: x quantised (with the whole sequence's scale), the
    fused in_proj, gates and q/k normalisation, the sequence-split scan, o
    quantised (whole-sequence scale), out_proj.  Every rank passes the same
    weights and ``state_in`` (None = zero).  Returns (y [B*T, hidden] for the
    local tokens, the quantised x, the quantised o, the state after the local
    span).  Collectives, in the same order on every rank: one max all-reduce
    (x), the scan's two all-gathers, one max all-reduce (o)."""
    ops = ops or CudaLayerOps()
    distributed = dist.is_initialized() and dist.get_world_size(group) > 1
    d = w.dims
    xq = _quantize_across(x, ops, group, distributed)
    P = ops.gemm(xq, w.w_in)
    q_hat, k_hat, v, g, beta = ops.gates(P, w)
    scale = 1.0 / float(d.K) ** 0.5
    o, S_end = sequence_parallel_scan(q_hat, k_hat, v, g, beta, B, T, d, scale=scale, form=form, state_in=state_in,
                                      group=group, ops=ops)
    oq = _quantize_across(o.reshape(B * T, d.Hv * d.V), ops, group, distributed)
    return ops.gemm(oq, w.w_out), xq, oq, S_end


def segmented_layer(w, xs, B: int, form: int = FORM_PAGES, state_in=None, ops=None):
    """sequence_parallel_layer's steps on one device, with the spans of every
    sequence given in order as a list of (x [B*T_i, hidden], T_i): the amax
    words of all spans first and their maximum in place of the all-reduce, then
    each span's in_proj and gates, the segmented scan, and the same for o.
    Returns the list of span outputs y and the final state."""
    ops = ops or CudaLayerOps()
    d = w.dims

    def quantize_all(ts):
        words = [ops.amax_word(t) for t in ts]
        word = torch.stack(words).amax(dim=0)
        return [ops.quantize_from_amax(t, word) for t in ts]

    xqs = quantize_all([x for x, _ in xs])
    spans = []
    for xq, (_, T) in zip(xqs, xs):
        q_hat, k_hat, v, g, beta = ops.gates(ops.gemm(xq, w.w_in), w)
        spans.append((q_hat, k_hat, v, g, beta, T))
    outs, S = segmented_scan(spans, B, d, scale=1.0 / float(d.K) ** 0.5, form=form, state_in=state_in, ops=ops)
    oqs = quantize_all([o.reshape(-1, d.Hv * d.V) for o in outs])
    return [ops.gemm(oq, w.w_out) for oq in oqs], xqs, oqs, S
