"""gdn_scan_noalloc: the allocation-free chunked scan for callers that cannot
allocate device memory (a host framework that owns every allocation, or code
that must not call cudaMalloc during CUDA-graph capture).  It runs the same
kernels as gdn_scan on the same inputs, so its output must equal the regular
gdn_scan's (which takes a caller-provided workspace) bit for bit, on two calls
in a row.  The second call also shows that what the first call left in the
shared scratch array does not leak into the result.  The small case is also
held to the scan bar against the oracle's recurrence.  Problems too large for
the fixed array must be refused up front; the largest accepted size follows
from the header's limit and gdn_scan_workspace_size, not from fixed numbers.

This file is named to be collected last.  It passes both when run alone in a
fresh process and after the rest of the suite."""
import ctypes

import numpy as np
import pytest
import torch

import gdn_synth
import nvfp4_w4a4_gated_b200 as nv
import oracle
from gpu_util import f32_device, rel_fro

pytestmark = pytest.mark.gpu

SCAN_TOL = 2e-3


def _inputs(seed, B, T, Hk, Hv, K, V):
    q, k, v, g, beta = gdn_synth.scan_inputs(seed, B, T, Hk, Hv, K, V, alpha_lo=0.8, alpha_hi=0.9999)
    S0 = gdn_synth.gaussian(seed + 1, (B, Hv, K, V), std=0.3)
    dev = (f32_device(q.reshape(B * T, Hk, K)), f32_device(k.reshape(B * T, Hk, K)),
           f32_device(v.reshape(B * T, Hv * V)), f32_device(g.reshape(B * T, Hv)),
           f32_device(beta.reshape(B * T, Hv)), f32_device(S0))
    return dev, (q, k, v, g, beta, S0)


def _scratch_bytes(B, T, dims):
    d = dims.c()
    return nv.lib().gdn_scan_workspace_size(B, T, ctypes.byref(d), nv.SCAN_CHUNKED)


@pytest.mark.parametrize("form", [nv.FORM_PAGES, nv.FORM_STANDARD])
def test_noalloc_scan_matches_workspace_scan_twice(cuda_dev, form):
    cases = [(1, 300, 16, 32, 128, 128, 3), (2, 130, 2, 4, 64, 128, 4)]   # two calls, different shapes
    for B, T, Hk, Hv, K, V, seed in cases:
        dims = nv.GdnDims(Hk, Hv, K, V)
        assert _scratch_bytes(B, T, dims) <= nv.NOALLOC_MAX_SCRATCH_BYTES
        (q, k, v, g, beta, S0), host = _inputs(seed, B, T, Hk, Hv, K, V)
        s_ref = torch.empty_like(S0)
        o_ref, _ = nv.gdn_scan(q, k, v, g, beta, B, T, dims, form=form, algo=nv.SCAN_CHUNKED, state_in=S0,
                               state_out=s_ref)
        s_na = torch.empty_like(S0)
        o_na, _ = nv.gdn_scan_noalloc(q, k, v, g, beta, B, T, dims, form=form, state_in=S0, state_out=s_na)
        torch.cuda.synchronize()
        nv.check_device_error()
        assert torch.equal(o_na, o_ref)
        assert torch.equal(s_na, s_ref)
        if T == 130:
            qh, kh, vh, gh, bh, S0h = host
            o_or, S_or = oracle.scan(qh, kh, vh, gh, bh, form=form, S0=S0h)
            assert rel_fro(o_na.cpu().numpy().reshape(o_or.shape), o_or) <= SCAN_TOL
            assert rel_fro(s_na.cpu().numpy(), S_or) <= SCAN_TOL


def test_noalloc_scan_refuses_oversize(cuda_dev):
    # B = 1, 32 value heads of 128 x 128: the largest T whose scratch fits the array
    # (found from gdn_scan_workspace_size, a whole chunk at a time) is accepted, one
    # chunk more is refused before anything is launched
    B, Hk, Hv, K, V = 1, 16, 32, 128, 128
    dims = nv.GdnDims(Hk, Hv, K, V)
    limit = nv.NOALLOC_MAX_SCRATCH_BYTES
    t_fit = 64
    while _scratch_bytes(B, t_fit + 64, dims) <= limit:
        t_fit += 64
    t_over = t_fit + 64
    assert _scratch_bytes(B, t_fit, dims) <= limit < _scratch_bytes(B, t_over, dims)
    (q, k, v, g, beta, _), _ = _inputs(5, B, t_over, Hk, Hv, K, V)
    with pytest.raises(nv.NVFP4Error) as ei:
        nv.gdn_scan_noalloc(q, k, v, g, beta, B, t_over, dims)
    assert ei.value.status == 6 and "scratch" in str(ei.value)
    o, _ = nv.gdn_scan_noalloc(q[:t_fit], k[:t_fit], v[:t_fit], g[:t_fit], beta[:t_fit], B, t_fit, dims)
    torch.cuda.synchronize()
    nv.check_device_error()
    assert torch.isfinite(o).all()
