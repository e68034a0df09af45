"""Thin Python binding of the sm_100a NVFP4 W4A4 Gated DeltaNet library.

Argument marshalling only: every step runs in the CUDA kernels of
``libnvfp4_gdn.so`` (built in-tree by ``nvfp4_w4a4_gated_b200.build``).  The
names mirror the C ABI in ``include/nvfp4_gdn.h``.  There is no CPU or PyTorch
fallback: if the library is missing, importing the binding's entry points
raises.  PyTorch is used only to own device memory and to name the stream.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import re

import torch

from . import build as _build

__all__ = [
    "NVFP4Error", "NVFP4Matrix", "GdnDims", "LayerWeights", "lib", "nvfp4_quantize", "w4a4_gemm", "gdn_gates",
    "gdn_scan", "gdn_scan_noalloc", "gdn_output_gate", "gdn_short_conv", "gdn_layer_forward", "layer_workspace_layout",
    "check_device_error", "gdn_scan_transition", "gdn_state_combine", "gdn_scan_correct", "gdn_scan_span",
    "selftest_wait_timeout", "FORM_PAGES",
    "FORM_STANDARD", "SCAN_AUTO", "SCAN_RECURRENT", "SCAN_CHUNKED", "EXPORTED_SYMBOLS", "QUANT_COMPUTE_SCALE",
    "QUANT_GIVEN_SCALE", "QUANT_AMAX_ONLY", "QUANT_FROM_AMAX",
]

FORM_PAGES, FORM_STANDARD = 0, 1
SCAN_AUTO, SCAN_RECURRENT, SCAN_CHUNKED = 0, 1, 2
DTYPE_BF16, DTYPE_FP32 = 0, 1
QUANT_COMPUTE_SCALE, QUANT_GIVEN_SCALE, QUANT_AMAX_ONLY, QUANT_FROM_AMAX = 0, 1, 2, 3

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED_SHAPE", 3: "MISALIGNED", 4: "CUDA", 5: "TIMEOUT", 6: "WORKSPACE"}

EXPORTED_SYMBOLS = [
    "nvfp4_last_error", "nvfp4_check_device_error", "nvfp4_version", "nvfp4_selftest_wait_timeout", "nvfp4_sf_bytes",
    "nvfp4_quantize_workspace_size", "nvfp4_quantize", "w4a4_gemm", "gdn_gates", "gdn_scan_workspace_size",
    "gdn_scan", "gdn_layer_workspace_layout", "gdn_layer_forward", "gdn_scan_noalloc", "gdn_output_gate",
    "gdn_short_conv", "gdn_layer_forward_stateful", "gdn_scan_transition_workspace_size", "gdn_scan_transition",
    "gdn_state_combine", "gdn_scan_correct", "gdn_scan_span_workspace_size", "gdn_scan_span",
    "gdn_layer_forward_timed",
]



def _header_size_macro(name: str) -> int:
    """Value of a `#define NAME ((size_t)A << B)` size macro of the C header."""
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nvfp4_gdn.h")
    m = re.search(r"#define\s+" + name + r"\s+\(\(size_t\)\s*(\d+)\s*<<\s*(\d+)\)", open(path).read())
    if m is None:
        raise RuntimeError(f"{name} not found in {path}")
    return int(m.group(1)) << int(m.group(2))


# Size of the fixed scratch array gdn_scan_noalloc uses, as the header defines it
# (GDN_SCAN_NOALLOC_MAX_SCRATCH_BYTES).
NOALLOC_MAX_SCRATCH_BYTES = _header_size_macro("GDN_SCAN_NOALLOC_MAX_SCRATCH_BYTES")


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class _Tensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("global_scale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class _Dims(ctypes.Structure):
    _fields_ = [("Hk", ctypes.c_int32), ("Hv", ctypes.c_int32), ("K", ctypes.c_int32), ("V", ctypes.c_int32)]


class _LayerWeights(ctypes.Structure):
    _fields_ = [("w_in", _Tensor), ("w_out", _Tensor), ("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
                ("dims", _Dims), ("hidden", ctypes.c_int32), ("out_norm", ctypes.c_void_p),
                ("conv_weight", ctypes.c_void_p), ("conv_width", ctypes.c_int32)]


_LAYOUT_FIELDS = ["x_codes", "x_sf", "x_scale", "proj", "q_hat", "k_hat", "g", "beta", "o", "o_gated", "qkv_conv",
                  "o_codes", "o_sf", "o_scale", "quant_ws", "scan_ws", "total"]


class _Layout(ctypes.Structure):
    _fields_ = [(f, ctypes.c_size_t) for f in _LAYOUT_FIELDS]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libnvfp4_gdn.so (building it first if the sources are newer)."""
    global _lib
    if _lib is None:
        path = _build.LIB
        if not os.path.exists(path) or not _build.up_to_date():
            path = _build.build()
        L = ctypes.CDLL(path)
        P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        TP = ctypes.POINTER(_Tensor)
        DP = ctypes.POINTER(_Dims)
        L.nvfp4_last_error.restype = ctypes.c_char_p
        L.nvfp4_version.restype = ctypes.c_char_p
        L.nvfp4_check_device_error.argtypes = [P]
        L.nvfp4_selftest_wait_timeout.argtypes = [ctypes.c_uint32, P]
        L.nvfp4_sf_bytes.argtypes = [i64, i64]
        L.nvfp4_sf_bytes.restype = sz
        L.nvfp4_quantize_workspace_size.restype = sz
        L.nvfp4_quantize.argtypes = [P, i32, i64, i64, i64, TP, i32, P, sz, P]
        L.w4a4_gemm.argtypes = [TP, TP, P, i64, P]
        L.gdn_gates.argtypes = [P, i64, i64, DP, P, P, P, P, P, P, P]
        L.gdn_output_gate.argtypes = [P, P, i64, P, i64, i32, i32, P, P, P]
        L.gdn_scan_workspace_size.argtypes = [i32, i64, DP, i32]
        L.gdn_scan_workspace_size.restype = sz
        L.gdn_scan.argtypes = [P, P, P, i64, P, P, i32, i64, DP, ctypes.c_float, i32, i32, P, P, P, P, sz, P]
        L.gdn_scan_noalloc.argtypes = [P, P, P, i64, P, P, i32, i64, DP, ctypes.c_float, i32, P, P, P, P]
        L.gdn_layer_workspace_layout.argtypes = [ctypes.POINTER(_LayerWeights), i32, i64, ctypes.POINTER(_Layout)]
        L.gdn_layer_forward.argtypes = [ctypes.POINTER(_LayerWeights), P, i32, i64, P, P, P, i32, P, sz, P]
        L.gdn_layer_forward_stateful.argtypes = [ctypes.POINTER(_LayerWeights), P, i32, i64, P, P, P, P, P, i32, P,
                                                 sz, P]
        L.gdn_layer_forward_timed.argtypes = [ctypes.POINTER(_LayerWeights), P, i32, i64, P, P, P, P, P, i32, P, sz,
                                              P, ctypes.POINTER(ctypes.c_void_p)]
        L.gdn_short_conv.argtypes = [P, i64, i32, i64, i32, i32, P, P, P, P, i64, P]
        L.gdn_scan_transition_workspace_size.argtypes = [i32, i64, DP, i32]
        L.gdn_scan_transition_workspace_size.restype = sz
        L.gdn_scan_transition.argtypes = [P, P, P, P, i32, i64, DP, ctypes.c_float, i32, i32, P, P, P, sz, P]
        L.gdn_state_combine.argtypes = [P, P, P, P, i32, i64, i32, i32, P]
        L.gdn_scan_span_workspace_size.argtypes = [i32, i64, DP, i32]
        L.gdn_scan_span_workspace_size.restype = sz
        L.gdn_scan_span.argtypes = [P, P, P, i64, P, P, i32, i64, DP, ctypes.c_float, i32, i32, P, P, P, P, P, sz, P]
        L.gdn_scan_correct.argtypes = [P, P, P, i32, i64, i32, i32, i32, P, P]
        for f in ("nvfp4_check_device_error", "nvfp4_selftest_wait_timeout", "nvfp4_quantize", "w4a4_gemm", "gdn_gates", "gdn_scan",
                  "gdn_layer_workspace_layout", "gdn_layer_forward", "gdn_scan_noalloc", "gdn_layer_forward_timed"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise NVFP4Error(status, lib().nvfp4_last_error().decode())


def _dev_addr(t) -> int:
    """Device address of a CUDA tensor; a host tensor is refused here, before
    any kernel could be handed a host pointer."""
    if not t.is_cuda:
        raise ValueError("the library takes CUDA tensors; got a tensor on " + str(t.device))
    return t.data_ptr()


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(_dev_addr(t))


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------------ tensors --
@dataclasses.dataclass
class NVFP4Matrix:
    """Device buffers of one NVFP4 matrix (codes, atom-layout scales, global scale)."""
    codes: torch.Tensor      # uint8 [rows, cols/2]
    sf: torch.Tensor         # uint8 [nvfp4_sf_bytes]
    scale: torch.Tensor      # float32 [1]
    rows: int
    cols: int

    @staticmethod
    def empty(rows: int, cols: int, device="cuda") -> "NVFP4Matrix":
        sf_bytes = lib().nvfp4_sf_bytes(rows, cols)
        return NVFP4Matrix(torch.empty((rows, cols // 2), dtype=torch.uint8, device=device),
                           torch.empty(sf_bytes, dtype=torch.uint8, device=device),
                           torch.empty(1, dtype=torch.float32, device=device), rows, cols)

    def c(self) -> _Tensor:
        return _Tensor(_dev_addr(self.codes), _dev_addr(self.sf), _dev_addr(self.scale), self.rows, self.cols)


@dataclasses.dataclass(frozen=True)
class GdnDims:
    Hk: int
    Hv: int
    K: int
    V: int

    def c(self) -> _Dims:
        return _Dims(self.Hk, self.Hv, self.K, self.V)

    @property
    def n_in(self) -> int:
        return 2 * self.Hk * self.K + 2 * self.Hv * self.V + 2 * self.Hv


@dataclasses.dataclass
class LayerWeights:
    w_in: NVFP4Matrix
    w_out: NVFP4Matrix
    A_log: torch.Tensor
    dt_bias: torch.Tensor
    dims: GdnDims
    hidden: int
    out_norm: torch.Tensor | None = None      # [V] weight of the optional output gate
    conv_weight: torch.Tensor | None = None   # [2 Hk K + Hv V, conv_width] optional short convolution
    conv_width: int = 4

    def c(self) -> _LayerWeights:
        return _LayerWeights(self.w_in.c(), self.w_out.c(), _dev_addr(self.A_log), _dev_addr(self.dt_bias),
                             self.dims.c(), self.hidden, _ptr(self.out_norm), _ptr(self.conv_weight),
                             self.conv_width)


def check_device_error(stream=None):
    _check(lib().nvfp4_check_device_error(_stream(stream)))


def selftest_wait_timeout(budget_cycles: int = 1 << 22, stream=None):
    """Exercise the bounded-wait failure path (see the C header)."""
    _check(lib().nvfp4_selftest_wait_timeout(budget_cycles, _stream(stream)))


# --------------------------------------------------------------- entry points --
_ws_cache = {}


def _scratch(nbytes: int, device) -> torch.Tensor:
    key = (str(device), "scratch")
    t = _ws_cache.get(key)
    if t is None or t.numel() < nbytes:
        t = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = t
    return t


def nvfp4_quantize(x: torch.Tensor, out: NVFP4Matrix | None = None, given_scale: bool = False, workspace=None,
                   stream=None, mode: int | None = None) -> NVFP4Matrix:
    """Quantise a bf16 or fp32 CUDA matrix to NVFP4 (the per-tensor scale is
    computed on the device unless ``given_scale``, which uses ``out.scale``).
    ``mode`` QUANT_AMAX_ONLY sets workspace word 0 to max|x| and writes nothing
    else; QUANT_FROM_AMAX quantises with S formed from workspace word 0 (for a
    tensor split across ranks: AMAX_ONLY, a max all-reduce of the word, then
    FROM_AMAX)."""
    assert x.is_cuda and x.dim() == 2 and x.stride(1) == 1
    dtype = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_FP32}[x.dtype]
    rows, cols = x.shape
    if out is None:
        out = NVFP4Matrix.empty(rows, cols, x.device)
    if workspace is None:
        workspace = _scratch(lib().nvfp4_quantize_workspace_size(), x.device)
    if mode is None:
        mode = QUANT_GIVEN_SCALE if given_scale else QUANT_COMPUTE_SCALE
    t = out.c()
    _check(lib().nvfp4_quantize(_ptr(x), dtype, rows, cols, x.stride(0), ctypes.byref(t), mode, _ptr(workspace),
                                workspace.numel(), _stream(stream)))
    return out


def w4a4_gemm(A: NVFP4Matrix, B: NVFP4Matrix, C: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """C = S_A S_B (A_hat @ B_hat^T), float32 [A.rows, B.rows]."""
    if C is None:
        C = torch.empty((A.rows, B.rows), dtype=torch.float32, device=A.codes.device)
    ta, tb = A.c(), B.c()
    _check(lib().w4a4_gemm(ctypes.byref(ta), ctypes.byref(tb), _ptr(C), C.stride(0), _stream(stream)))
    return C


def gdn_gates(proj: torch.Tensor, dims: GdnDims, A_log: torch.Tensor, dt_bias: torch.Tensor, stream=None):
    """Returns (q_hat [n,Hk,K], k_hat [n,Hk,K], g [n,Hv], beta [n,Hv]) from the fused projection."""
    n = proj.shape[0]
    dev = proj.device
    q_hat = torch.empty((n, dims.Hk, dims.K), dtype=torch.float32, device=dev)
    k_hat = torch.empty_like(q_hat)
    g = torch.empty((n, dims.Hv), dtype=torch.float32, device=dev)
    beta = torch.empty_like(g)
    d = dims.c()
    _check(lib().gdn_gates(_ptr(proj), proj.stride(0), n, ctypes.byref(d), _ptr(A_log), _ptr(dt_bias), _ptr(q_hat),
                           _ptr(k_hat), _ptr(g), _ptr(beta), _stream(stream)))
    return q_hat, k_hat, g, beta


def gdn_output_gate(o: torch.Tensor, z: torch.Tensor, w: torch.Tensor, out=None, amax_word=None, stream=None):
    """Output gate: out = o / sqrt(mean(o^2) + 1e-6) * w * SiLU(z) per (token, value
    head).  o: [n, Hv, V] contiguous; z: a [n, >= Hv*V] view (row stride ld_z);
    w: [V].  Returns out (a new tensor unless given; may be o)."""
    n, Hv, V = o.shape
    if out is None:
        out = torch.empty_like(o)
    _check(lib().gdn_output_gate(_ptr(o), _ptr(z), z.stride(0), _ptr(w), n, Hv, V, _ptr(out), _ptr(amax_word),
                                 _stream(stream)))
    return out


def gdn_short_conv(x: torch.Tensor, w: torch.Tensor, B: int, T: int, out=None, state_in=None, state_out=None,
                   stream=None):
    """Short causal convolution + SiLU per channel.  x: a [B*T, >= C] view (row
    stride ld_x); w: [C, W]; state_in / state_out: [B, C, W-1] or None.
    Returns out [B*T, C] (a new tensor unless given)."""
    C, W = w.shape
    if out is None:
        out = torch.empty((B * T, C), dtype=torch.float32, device=x.device)
    _check(lib().gdn_short_conv(_ptr(x), x.stride(0), B, T, C, W, _ptr(w), _ptr(state_in), _ptr(state_out), _ptr(out),
                                out.stride(0), _stream(stream)))
    return out


def gdn_scan(q_hat, k_hat, v, g, beta, B: int, T: int, dims: GdnDims, scale: float | None = None,
             form: int = FORM_PAGES, algo: int = SCAN_AUTO, state_in=None, state_out=None, o=None,
             workspace=None, stream=None):
    """Delta-rule scan.  q_hat/k_hat [B*T, Hk, K]; v a [B*T, >=Hv*V] view (row
    stride ld_v); g, beta [B*T, Hv].  Returns (o [B*T, Hv, V], state_out)."""
    dev = q_hat.device
    if scale is None:
        scale = 1.0 / math.sqrt(dims.K)
    if o is None:
        o = torch.empty((B * T, dims.Hv, dims.V), dtype=torch.float32, device=dev)
    d = dims.c()
    need = lib().gdn_scan_workspace_size(B, T, ctypes.byref(d), algo)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ld_v = v.stride(0)
    _check(lib().gdn_scan(_ptr(q_hat), _ptr(k_hat), _ptr(v), ld_v, _ptr(g), _ptr(beta), B, T, ctypes.byref(d),
                          float(scale), form, algo, _ptr(state_in), _ptr(state_out), _ptr(o), _ptr(workspace),
                          0 if workspace is None else workspace.numel(), _stream(stream)))
    return o, state_out


def gdn_scan_transition(q_hat, k_hat, g, beta, B: int, T: int, dims: GdnDims, scale: float | None = None,
                        form: int = FORM_PAGES, algo: int = SCAN_AUTO, P=None, qmap=None, workspace=None,
                        stream=None):
    """Span map P [B, Hv, K, K] and query map [B*T, Hv, K] of B spans of T
    tokens: a span started from S_in ends in P S_in + S_loc and its outputs
    gain S_in^T qmap_t.  Inputs as for gdn_scan."""
    dev = q_hat.device
    if scale is None:
        scale = 1.0 / math.sqrt(dims.K)
    if P is None:
        P = torch.empty((B, dims.Hv, dims.K, dims.K), dtype=torch.float32, device=dev)
    if qmap is None:
        qmap = torch.empty((B * T, dims.Hv, dims.K), dtype=torch.float32, device=dev)
    d = dims.c()
    need = lib().gdn_scan_transition_workspace_size(B, T, ctypes.byref(d), algo)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check(lib().gdn_scan_transition(_ptr(q_hat), _ptr(k_hat), _ptr(g), _ptr(beta), B, T, ctypes.byref(d),
                                     float(scale), form, algo, _ptr(P), _ptr(qmap), _ptr(workspace),
                                     workspace.numel(), _stream(stream)))
    return P, qmap


def gdn_state_combine(P, S_loc, S_in, out=None, stream=None):
    """The maps of m spans composed in order: S = S_in, then S = P[j] S +
    S_loc[j] for each j; returns S [B, Hv, K, V].  P [m, B, Hv, K, K] (or
    [B, Hv, K, K]: one step), S_loc shaped like P with V columns (None = zero),
    S_in [B, Hv, K, V] (None = zero).  out may be S_in."""
    B, Hv, K = P.shape[-4], P.shape[-3], P.shape[-1]
    n = B * Hv
    m = P.numel() // (n * K * K)
    V = (S_in if S_in is not None else S_loc).shape[-1]
    if out is None:
        out = torch.empty((B, Hv, K, V), dtype=torch.float32, device=P.device)
    _check(lib().gdn_state_combine(_ptr(P), _ptr(S_loc), _ptr(S_in), _ptr(out), m, n, K, V, _stream(stream)))
    return out


def gdn_scan_span(q_hat, k_hat, v, g, beta, B: int, T: int, dims: GdnDims, scale: float | None = None,
                  form: int = FORM_PAGES, algo: int = SCAN_AUTO, workspace=None, stream=None):
    """A span's zero-start scan and its maps in one call: returns (o [B*T, Hv, V],
    S_loc [B, Hv, K, V], P [B, Hv, K, K], qmap [B*T, Hv, K])."""
    dev = q_hat.device
    if scale is None:
        scale = 1.0 / math.sqrt(dims.K)
    f32 = dict(dtype=torch.float32, device=dev)
    o = torch.empty((B * T, dims.Hv, dims.V), **f32)
    S_loc = torch.empty((B, dims.Hv, dims.K, dims.V), **f32)
    P = torch.empty((B, dims.Hv, dims.K, dims.K), **f32)
    qmap = torch.empty((B * T, dims.Hv, dims.K), **f32)
    d = dims.c()
    need = lib().gdn_scan_span_workspace_size(B, T, ctypes.byref(d), algo)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check(lib().gdn_scan_span(_ptr(q_hat), _ptr(k_hat), _ptr(v), v.stride(0), _ptr(g), _ptr(beta), B, T,
                               ctypes.byref(d), float(scale), form, algo, _ptr(o), _ptr(S_loc), _ptr(P), _ptr(qmap),
                               _ptr(workspace), workspace.numel(), _stream(stream)))
    return o, S_loc, P, qmap


def gdn_scan_correct(qmap, S_in, o, B: int, T: int, amax_word=None, stream=None):
    """o += S_in^T qmap per (sequence, token, value head), in place: qmap
    [B*T, Hv, K], S_in [B, Hv, K, V], o [B*T, Hv, V]."""
    Hv, K, V = S_in.shape[1], S_in.shape[2], S_in.shape[3]
    _check(lib().gdn_scan_correct(_ptr(qmap), _ptr(S_in), _ptr(o), B, T, Hv, K, V, _ptr(amax_word),
                                  _stream(stream)))
    return o


def gdn_scan_noalloc(q_hat, k_hat, v, g, beta, B: int, T: int, dims: GdnDims, scale: float | None = None,
                     form: int = FORM_PAGES, state_in=None, state_out=None, o=None, stream=None):
    """Chunked scan with the library's own fixed scratch array (no workspace
    argument, nothing allocated by the library)."""
    dev = q_hat.device
    if scale is None:
        scale = 1.0 / math.sqrt(dims.K)
    if o is None:
        o = torch.empty((B * T, dims.Hv, dims.V), dtype=torch.float32, device=dev)
    d = dims.c()
    _check(lib().gdn_scan_noalloc(_ptr(q_hat), _ptr(k_hat), _ptr(v), v.stride(0), _ptr(g), _ptr(beta), B, T,
                                  ctypes.byref(d), float(scale), form, _ptr(state_in), _ptr(state_out), _ptr(o),
                                  _stream(stream)))
    return o, state_out


def layer_workspace_layout(w: LayerWeights, B: int, T: int) -> dict:
    lw = w.c()
    L = _Layout()
    _check(lib().gdn_layer_workspace_layout(ctypes.byref(lw), B, T, ctypes.byref(L)))
    return {f: getattr(L, f) for f in _LAYOUT_FIELDS}


def gdn_layer_forward(w: LayerWeights, x: torch.Tensor, B: int, T: int, y=None, state_in=None, state_out=None,
                      form: int = FORM_PAGES, workspace=None, stream=None, conv_state_in=None, conv_state_out=None,
                      events=None):
    """y = GDN layer(x) under NVFP4 W4A4.  x: bf16 [B*T, hidden] on the device.
    conv_state_in / conv_state_out: the short convolution's carried inputs
    [B, 2 Hk K + Hv V, conv_width - 1] (used only when w.conv_weight is set).
    events: optional list of 7 torch.cuda.Event (timing enabled), recorded on the
    stream around the layer's stages (gdn_layer_forward_timed)."""
    assert x.dtype == torch.bfloat16 and x.is_contiguous()
    if y is None:
        y = torch.empty((B * T, w.hidden), dtype=torch.float32, device=x.device)
    lay = layer_workspace_layout(w, B, T)
    if workspace is None:
        workspace = torch.empty(lay["total"], dtype=torch.uint8, device=x.device)
    lw = w.c()
    if events is not None:
        if len(events) != 7:
            raise ValueError("events: 7 torch.cuda.Event")
        st = stream if stream is not None else torch.cuda.current_stream(x.device)
        for ev in events:
            if ev.cuda_event == 0:   # torch creates the CUDA event on its first record
                ev.record(st)
        handles = (ctypes.c_void_p * 7)(*[ev.cuda_event for ev in events])
        _check(lib().gdn_layer_forward_timed(ctypes.byref(lw), _ptr(x), B, T, _ptr(y), _ptr(state_in),
                                             _ptr(state_out), _ptr(conv_state_in), _ptr(conv_state_out), form,
                                             _ptr(workspace), workspace.numel(), _stream(st), handles))
        return y, workspace, lay
    _check(lib().gdn_layer_forward_stateful(ctypes.byref(lw), _ptr(x), B, T, _ptr(y), _ptr(state_in), _ptr(state_out),
                                            _ptr(conv_state_in), _ptr(conv_state_out), form, _ptr(workspace),
                                            workspace.numel(), _stream(stream)))
    return y, workspace, lay
