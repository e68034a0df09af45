"""The C-ABI library loads, exports every symbol the header declares, and its
host-side validation rejects bad arguments before launching anything.  CPU only:
no call here reaches a kernel launch."""
import ctypes
import re
import os

import pytest

import nvfp4_w4a4_gated_b200 as nv
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "nvfp4_gdn.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


def test_header_declares_the_binding_symbols():
    assert declared_symbols() == sorted(nv.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    L = nv.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_version_and_sizes():
    L = nv.lib()
    assert L.nvfp4_version().decode().count(".") == 2
    assert L.nvfp4_sf_bytes(1, 64) == 128 * 4
    assert L.nvfp4_sf_bytes(129, 128) == 256 * 8
    assert L.nvfp4_sf_bytes(8192, 5120) == 8192 * 320
    assert L.nvfp4_quantize_workspace_size() >= 4
    d = nv.GdnDims(16, 32, 128, 128).c()
    assert L.gdn_scan_workspace_size(1, 1, ctypes.byref(d), nv.SCAN_AUTO) == 0
    n = L.gdn_scan_workspace_size(1, 4096, ctypes.byref(d), nv.SCAN_CHUNKED)
    assert n >= 32 * 64 * (64 * 128 * 2 + 64 * 64 + 64) * 4
    bad = nv.GdnDims(3, 32, 128, 128).c()
    assert L.gdn_scan_workspace_size(1, 4096, ctypes.byref(bad), nv.SCAN_CHUNKED) == 0


def _err(status):
    return status, nv.lib().nvfp4_last_error().decode()


FAKE = 0x10000  # a 16-byte aligned non-null address; never dereferenced (validation fails first)


def _tensor(rows=128, cols=256, codes=FAKE, sf=FAKE, scale=FAKE):
    return nv._Tensor(codes, sf, scale, rows, cols)


def test_quantize_validation():
    L = nv.lib()
    t = _tensor()
    st, msg = _err(L.nvfp4_quantize(None, 0, 128, 256, 256, ctypes.byref(t), 0, FAKE, 256, None))
    assert st == 1 and "null" in msg
    st, _ = _err(L.nvfp4_quantize(FAKE, 7, 128, 256, 256, ctypes.byref(t), 0, FAKE, 256, None))
    assert st == 1
    t2 = _tensor(cols=100)
    st, _ = _err(L.nvfp4_quantize(FAKE, 0, 128, 100, 100, ctypes.byref(t2), 0, FAKE, 256, None))
    assert st == 2
    st, _ = _err(L.nvfp4_quantize(FAKE + 2, 0, 128, 256, 256, ctypes.byref(t), 0, FAKE, 256, None))
    assert st == 3
    st, _ = _err(L.nvfp4_quantize(FAKE, 0, 128, 256, 256, ctypes.byref(t), 0, None, 0, None))
    assert st == 6
    st, _ = _err(L.nvfp4_quantize(FAKE, 0, 64, 256, 256, ctypes.byref(t), 0, FAKE, 256, None))
    assert st == 1  # shape differs from out
    st, _ = _err(L.nvfp4_quantize(FAKE, 0, 128, 256, 256, ctypes.byref(t), 4, FAKE, 256, None))
    assert st == 1  # unknown flag
    for flag in (nv.QUANT_AMAX_ONLY, nv.QUANT_FROM_AMAX):   # the word lives in the workspace
        st, _ = _err(L.nvfp4_quantize(FAKE, 0, 128, 256, 256, ctypes.byref(t), flag, None, 0, None))
        assert st == 6


def test_gemm_validation():
    L = nv.lib()
    A, B = _tensor(128, 256), _tensor(64, 512)
    st, msg = _err(L.w4a4_gemm(ctypes.byref(A), ctypes.byref(B), FAKE, 64, None))
    assert st == 1 and "K" in msg
    B = _tensor(66, 256)
    st, _ = _err(L.w4a4_gemm(ctypes.byref(A), ctypes.byref(B), FAKE, 68, None))
    assert st == 2
    B = _tensor(64, 256)
    st, _ = _err(L.w4a4_gemm(ctypes.byref(A), ctypes.byref(B), FAKE, 62, None))
    assert st == 1
    st, _ = _err(L.w4a4_gemm(ctypes.byref(A), ctypes.byref(B), FAKE + 4, 64, None))
    assert st == 3
    A = _tensor(128, 256, codes=FAKE + 8)
    st, _ = _err(L.w4a4_gemm(ctypes.byref(A), ctypes.byref(B), FAKE, 64, None))
    assert st == 3
    A = _tensor(128, 256, sf=0)
    st, _ = _err(L.w4a4_gemm(ctypes.byref(A), ctypes.byref(B), FAKE, 64, None))
    assert st == 1


def test_gates_and_scan_validation():
    L = nv.lib()
    d = nv.GdnDims(16, 32, 128, 128).c()
    n_in = 2 * 16 * 128 + 2 * 32 * 128 + 64
    st, _ = _err(L.gdn_gates(FAKE, n_in - 4, 10, ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None))
    assert st == 1
    bad = nv.GdnDims(16, 32, 96, 128).c()
    st, _ = _err(L.gdn_gates(FAKE, n_in, 10, ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None))
    assert st == 2
    st, _ = _err(L.gdn_scan(FAKE, FAKE, FAKE, 4096, FAKE, FAKE, 1, 64, ctypes.byref(d), 0.1, 5, 0, None, None, FAKE,
                            FAKE, 1 << 30, None))
    assert st == 1
    st, _ = _err(L.gdn_scan(FAKE, FAKE, FAKE, 4096, FAKE, FAKE, 1, 4096, ctypes.byref(d), 0.1, 0, 2, None, None, FAKE,
                            None, 0, None))
    assert st == 6
    st, _ = _err(L.gdn_scan(FAKE, FAKE, FAKE, 100, FAKE, FAKE, 1, 64, ctypes.byref(d), 0.1, 0, 0, None, None, FAKE,
                            FAKE, 1 << 30, None))
    assert st == 1


def test_scan_refuses_unaligned_state_pointers():
    """The chunked scan moves the state as 16-byte vectors: an offset state_in or
    state_out is refused on the host (MISALIGNED), for gdn_scan, the
    allocation-free variant and the layer."""
    L = nv.lib()
    d = nv.GdnDims(16, 32, 128, 128).c()
    for s_in, s_out in ((FAKE + 4, None), (None, FAKE + 8), (FAKE + 4, FAKE + 4)):
        st, msg = _err(L.gdn_scan(FAKE, FAKE, FAKE, 4096, FAKE, FAKE, 1, 64, ctypes.byref(d), 0.1, 0, 2, s_in, s_out,
                                  FAKE, FAKE, 1 << 30, None))
        assert st == 3 and "state" in msg
        st, msg = _err(L.gdn_scan_noalloc(FAKE, FAKE, FAKE, 4096, FAKE, FAKE, 1, 64, ctypes.byref(d), 0.1, 0, s_in,
                                          s_out, FAKE, None))
        assert st == 3 and "state" in msg
    dims = nv.GdnDims(16, 32, 128, 128)
    lw = nv._LayerWeights(_tensor(dims.n_in, 5120), _tensor(5120, 4096), FAKE, FAKE, dims.c(), 5120)
    st, msg = _err(L.gdn_layer_forward(ctypes.byref(lw), FAKE, 1, 64, FAKE, FAKE + 4, None, 0, FAKE, 1 << 40, None))
    assert st == 3 and "state" in msg


def test_layer_layout_and_validation():
    L = nv.lib()
    dims = nv.GdnDims(16, 32, 128, 128)
    w_in = nv.NVFP4Matrix(None, None, None, dims.n_in, 5120)
    lw = nv._LayerWeights(_tensor(dims.n_in, 5120), _tensor(5120, 4096), FAKE, FAKE, dims.c(), 5120)
    lay = nv._Layout()
    assert L.gdn_layer_workspace_layout(ctypes.byref(lw), 1, 4096, ctypes.byref(lay)) == 0
    assert lay.proj > lay.x_scale and lay.total > lay.scan_ws
    assert all(getattr(lay, f) % 256 == 0 for f in nv._LAYOUT_FIELDS)
    assert lay.q_hat - lay.proj >= 4096 * 12352 * 4
    lw_bad = nv._LayerWeights(_tensor(dims.n_in - 64, 5120), _tensor(5120, 4096), FAKE, FAKE, dims.c(), 5120)
    st, msg = _err(L.gdn_layer_workspace_layout(ctypes.byref(lw_bad), 1, 4096, ctypes.byref(lay)))
    assert st == 1 and "w_in" in msg
    st, _ = _err(L.gdn_layer_forward(ctypes.byref(lw), FAKE, 1, 4096, FAKE, None, None, 0, FAKE, 10, None))
    assert st == 6
    st, _ = _err(L.gdn_layer_forward(ctypes.byref(lw), FAKE, 1, 4096, FAKE, None, None, 3, FAKE, 1 << 40, None))
    assert st == 1
    # the timed variant checks its seven event handles before anything else
    st, msg = _err(L.gdn_layer_forward_timed(ctypes.byref(lw), FAKE, 1, 4096, FAKE, None, None, None, None, 0, FAKE,
                                             1 << 40, None, None))
    assert st == 1 and "events" in msg
    handles = (ctypes.c_void_p * 7)(*([FAKE] * 6 + [None]))
    st, msg = _err(L.gdn_layer_forward_timed(ctypes.byref(lw), FAKE, 1, 4096, FAKE, None, None, None, None, 0, FAKE,
                                             1 << 40, None, handles))
    assert st == 1 and "event" in msg
    del w_in


def test_selftest_budget_validation():
    L = nv.lib()
    for budget in (0, (1 << 30) + 1):
        st, msg = _err(L.nvfp4_selftest_wait_timeout(budget, None))
        assert st == 1 and "budget" in msg


def test_output_gate_validation_and_layout():
    L = nv.lib()
    st, _ = _err(L.gdn_output_gate(None, FAKE, 4096, FAKE, 10, 32, 128, FAKE, None, None))
    assert st == 1
    st, _ = _err(L.gdn_output_gate(FAKE, FAKE, 4096, FAKE, 10, 32, 96, FAKE, None, None))
    assert st == 2
    st, _ = _err(L.gdn_output_gate(FAKE, FAKE, 4000, FAKE, 10, 32, 128, FAKE, None, None))
    assert st == 1
    st, _ = _err(L.gdn_output_gate(FAKE, FAKE, 4098, FAKE, 10, 32, 128, FAKE, None, None))
    assert st == 3
    # the layout reserves a gated-output region only when the gate weight is set
    dims = nv.GdnDims(16, 32, 128, 128)
    lay0, lay1 = nv._Layout(), nv._Layout()
    lw0 = nv._LayerWeights(_tensor(dims.n_in, 5120), _tensor(5120, 4096), FAKE, FAKE, dims.c(), 5120, None)
    lw1 = nv._LayerWeights(_tensor(dims.n_in, 5120), _tensor(5120, 4096), FAKE, FAKE, dims.c(), 5120, FAKE)
    assert L.gdn_layer_workspace_layout(ctypes.byref(lw0), 1, 4096, ctypes.byref(lay0)) == 0
    assert L.gdn_layer_workspace_layout(ctypes.byref(lw1), 1, 4096, ctypes.byref(lay1)) == 0
    assert lay0.o_codes == lay0.o_gated and lay1.o_codes - lay1.o_gated >= 4096 * 4096 * 4
    assert lay1.total - lay0.total == lay1.o_codes - lay1.o_gated


def test_short_conv_validation_and_layout():
    L = nv.lib()
    st, _ = _err(L.gdn_short_conv(None, 8192, 1, 64, 8192, 4, FAKE, None, None, FAKE, 8192, None))
    assert st == 1
    st, _ = _err(L.gdn_short_conv(FAKE, 8192, 1, 64, 8192, 5, FAKE, None, None, 0x4000000, 8192, None))
    assert st == 2
    st, msg = _err(L.gdn_short_conv(FAKE, 8192, 1, 64, 8192, 4, FAKE, None, None, FAKE + 4096, 8192, None))
    assert st == 1 and "overlap" in msg
    dims = nv.GdnDims(16, 32, 128, 128)
    C = 2 * 16 * 128 + 32 * 128
    lay0, lay1 = nv._Layout(), nv._Layout()
    lw0 = nv._LayerWeights(_tensor(dims.n_in, 5120), _tensor(5120, 4096), FAKE, FAKE, dims.c(), 5120, None, None, 4)
    lw1 = nv._LayerWeights(_tensor(dims.n_in, 5120), _tensor(5120, 4096), FAKE, FAKE, dims.c(), 5120, None, FAKE, 4)
    assert L.gdn_layer_workspace_layout(ctypes.byref(lw0), 1, 4096, ctypes.byref(lay0)) == 0
    assert L.gdn_layer_workspace_layout(ctypes.byref(lw1), 1, 4096, ctypes.byref(lay1)) == 0
    assert lay1.o_codes - lay1.qkv_conv >= 4096 * C * 4 and lay0.o_codes == lay0.qkv_conv
    lw_bad = nv._LayerWeights(_tensor(dims.n_in, 5120), _tensor(5120, 4096), FAKE, FAKE, dims.c(), 5120, None, FAKE, 7)
    st, msg = _err(L.gdn_layer_workspace_layout(ctypes.byref(lw_bad), 1, 4096, ctypes.byref(lay1)))
    assert st == 2 and "conv_width" in msg


def test_state_passing_validation_and_sizes():
    L = nv.lib()
    d = nv.GdnDims(16, 32, 128, 64).c()
    # the transition runs the scan with V = K plus one zero row of Hv*K floats
    dk = nv.GdnDims(16, 32, 128, 128).c()
    scan_ws = L.gdn_scan_workspace_size(1, 4096, ctypes.byref(dk), nv.SCAN_CHUNKED)
    tw = L.gdn_scan_transition_workspace_size(1, 4096, ctypes.byref(d), nv.SCAN_CHUNKED)
    assert tw >= scan_ws + 32 * 128 * 4 and tw % 256 == 0
    assert L.gdn_scan_transition_workspace_size(1, 1, ctypes.byref(d), nv.SCAN_AUTO) == 256 * ((32 * 128 * 4 + 255) // 256)
    big = 0x40000000
    st, _ = _err(L.gdn_scan_transition(None, FAKE, FAKE, FAKE, 1, 64, ctypes.byref(d), 1.0, 0, 0, FAKE, FAKE,
                                       FAKE, 1 << 30, None))
    assert st == 1
    st, msg = _err(L.gdn_scan_transition(FAKE, FAKE, FAKE, FAKE, 1, 4096, ctypes.byref(d), 1.0, 0, 2, big,
                                         2 * big, 3 * big, tw - 1, None))
    assert st == 6
    st, msg = _err(L.gdn_scan_transition(FAKE, FAKE, FAKE, FAKE, 1, 4096, ctypes.byref(d), 1.0, 0, 2, big, big,
                                         3 * big, tw, None))
    assert st == 1 and "overlap" in msg
    st, _ = _err(L.gdn_scan_transition(FAKE, FAKE, FAKE, FAKE, 1, 64, ctypes.byref(d), 1.0, 5, 0, big, 2 * big,
                                       3 * big, tw, None))
    assert st == 1
    # combine (a chain of m maps): shapes, aliasing
    st, _ = _err(L.gdn_state_combine(FAKE, FAKE, FAKE, None, 1, 4, 128, 128, None))
    assert st == 1
    st, _ = _err(L.gdn_state_combine(FAKE, FAKE, FAKE, big, 0, 4, 128, 128, None))
    assert st == 1
    st, _ = _err(L.gdn_state_combine(FAKE, FAKE, FAKE, big, 1, 4, 48, 128, None))
    assert st == 2
    st, _ = _err(L.gdn_state_combine(FAKE, FAKE, FAKE, big, 1, 4, 256, 128, None))
    assert st == 2
    st, _ = _err(L.gdn_state_combine(FAKE, FAKE, FAKE, big, 1, 4, 128, 100, None))
    assert st == 2
    st, _ = _err(L.gdn_state_combine(FAKE + 4, FAKE, FAKE, big, 1, 4, 128, 128, None))
    assert st == 3
    st, msg = _err(L.gdn_state_combine(big, 2 * big, 3 * big, 3 * big + 4096, 1, 4, 128, 128, None))
    assert st == 1 and "S_in" in msg
    sb = 4 * 128 * 128 * 4          # one state block of n = 4
    st, msg = _err(L.gdn_state_combine(big, 2 * big, 3 * big, 2 * big, 3, 4, 128, 128, None))
    assert st == 1 and "S_loc" in msg
    st, msg = _err(L.gdn_state_combine(big, 2 * big, 3 * big, big + 1024, 1, 4, 128, 128, None))
    assert st == 1 and "P" in msg
    # the span step
    tws = L.gdn_scan_span_workspace_size(1, 4096, ctypes.byref(dk), nv.SCAN_CHUNKED)
    assert tws >= max(scan_ws, L.gdn_scan_transition_workspace_size(1, 4096, ctypes.byref(dk), nv.SCAN_CHUNKED))
    st, _ = _err(L.gdn_scan_span(FAKE, FAKE, FAKE, 4096, FAKE, FAKE, 1, 4096, ctypes.byref(dk), 1.0, 0, 0, None,
                                 big, 2 * big, 3 * big, 4 * big, tws, None))
    assert st == 1
    st, _ = _err(L.gdn_scan_span(FAKE, FAKE, FAKE, 4096, FAKE, FAKE, 1, 4096, ctypes.byref(dk), 1.0, 0, 0, big,
                                 2 * big, 3 * big, 4 * big, 5 * big, tws - 1, None))
    assert st == 6
    st, msg = _err(L.gdn_scan_span(FAKE, FAKE, FAKE, 4096, FAKE, FAKE, 1, 4096, ctypes.byref(dk), 1.0, 0, 0, big,
                                   big + 4096, 3 * big, 4 * big, 5 * big, tws, None))
    assert st == 1 and "overlap" in msg
    assert sb > 0
    # correct: head dims, alignment, aliasing
    st, _ = _err(L.gdn_scan_correct(FAKE, FAKE, big, 1, 64, 32, 96, 128, None, None))
    assert st == 2
    st, _ = _err(L.gdn_scan_correct(FAKE + 4, FAKE, big, 1, 64, 32, 128, 128, None, None))
    assert st == 3
    st, msg = _err(L.gdn_scan_correct(big, 2 * big, big + 4096, 1, 64, 32, 128, 128, None, None))
    assert st == 1 and "overlap" in msg
    st, _ = _err(L.gdn_scan_correct(FAKE, FAKE, big, 70000, 64, 32, 128, 128, None, None))
    assert st == 2


def test_binding_refuses_host_tensors():
    """A CPU tensor never reaches the library as a pointer: the binding raises
    on the host before any call (on a machine with a GPU a host pointer in a kernel would
    fault)."""
    import torch
    import pytest as _pytest
    x = torch.zeros((64, 128), dtype=torch.float32)
    with _pytest.raises(ValueError, match="CUDA tensors"):
        nv._ptr(x)
    S = torch.zeros((1, 2, 64, 64))
    with _pytest.raises(ValueError, match="CUDA tensors"):
        nv.gdn_state_combine(torch.zeros((1, 2, 64, 64)), S, S)
    m = nv.NVFP4Matrix(torch.zeros((64, 32), dtype=torch.uint8), torch.zeros(512, dtype=torch.uint8),
                       torch.zeros(1), 64, 64)
    with _pytest.raises(ValueError, match="CUDA tensors"):
        m.c()
