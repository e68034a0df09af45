"""gdn_scan_noalloc: the allocation-free chunked scan for callers that cannot
allocate device memory (a host framework that owns every allocation, or code
that must not call cudaMalloc during CUDA-graph capture).  Its output must match
the regular gdn_scan, which takes a caller-provided workspace, on two calls in a
row.  The second call also checks that the contents the first call left in the
shared scratch array do not leak into the result.  Problems too large for the
fixed array must be refused up front.

This file is named to be collected last.  It passes both when run alone in a
fresh process and after the rest of the suite."""
import numpy as np
import pytest
import torch

import gdn_synth
import nvfp4_w4a4_gated_b200 as nv
from gpu_util import f32_device, rel_fro

pytestmark = pytest.mark.gpu

SCAN_TOL = 2e-3


def _inputs(seed, B, T, Hk, Hv, K, V):
    q, k, v, g, beta = gdn_synth.scan_inputs(seed, B, T, Hk, Hv, K, V, alpha_lo=0.8, alpha_hi=0.9999)
    S0 = gdn_synth.gaussian(seed + 1, (B, Hv, K, V), std=0.3)
    return (f32_device(q.reshape(B * T, Hk, K)), f32_device(k.reshape(B * T, Hk, K)),
            f32_device(v.reshape(B * T, Hv * V)), f32_device(g.reshape(B * T, Hv)),
            f32_device(beta.reshape(B * T, Hv)), f32_device(S0))


@pytest.mark.parametrize("form", [nv.FORM_PAGES, nv.FORM_STANDARD])
def test_noalloc_scan_matches_workspace_scan_twice(cuda_dev, form):
    cases = [(1, 800, 16, 32, 128, 128, 3), (2, 130, 2, 4, 64, 128, 4)]   # two calls, different shapes
    for B, T, Hk, Hv, K, V, seed in cases:
        dims = nv.GdnDims(Hk, Hv, K, V)
        q, k, v, g, beta, S0 = _inputs(seed, B, T, Hk, Hv, K, V)
        s_ref = torch.empty_like(S0)
        o_ref, _ = nv.gdn_scan(q, k, v, g, beta, B, T, dims, form=form, algo=nv.SCAN_CHUNKED, state_in=S0,
                               state_out=s_ref)
        s_na = torch.empty_like(S0)
        o_na, _ = nv.gdn_scan_noalloc(q, k, v, g, beta, B, T, dims, form=form, state_in=S0, state_out=s_na)
        torch.cuda.synchronize()
        nv.check_device_error()
        assert rel_fro(o_na.cpu().numpy(), o_ref.cpu().numpy()) <= SCAN_TOL
        assert rel_fro(s_na.cpu().numpy(), s_ref.cpu().numpy()) <= SCAN_TOL
        assert torch.isfinite(o_na).all()


def test_noalloc_scan_refuses_oversize(cuda_dev):
    # B = 1, 32 value heads of 128 x 128: 896 tokens fit in the 64 MiB array, 960 do not
    B, Hk, Hv, K, V = 1, 16, 32, 128, 128
    dims = nv.GdnDims(Hk, Hv, K, V)
    q, k, v, g, beta, S0 = _inputs(5, B, 960, Hk, Hv, K, V)
    with pytest.raises(nv.NVFP4Error) as ei:
        nv.gdn_scan_noalloc(q, k, v, g, beta, B, 960, dims)
    assert ei.value.status == 6 and "scratch" in str(ei.value)
    o, _ = nv.gdn_scan_noalloc(q[:896], k[:896], v[:896], g[:896], beta[:896], B, 896, dims)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all()
    assert nv.NOALLOC_MAX_SCRATCH_BYTES == 64 << 20
