"""CPU oracle for the NVFP4 W4A4 Gated DeltaNet layer forward.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product library
never does, and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C: exact float32 for the
quantiser, float64 elsewhere); this module only marshals numpy arrays and
composes the steps in the order the pages give them:

1. online NVFP4 quantisation of the activations (review page "Why Gated
   DeltaNet Survives 4-Bit Quantization", background / paper sec.1);
2. block-scaled FP4 x FP4 GEMM for the fused q|k|v|z|a|b projection with one
   harmonised weight scale (review page, paper sec.6; abstract page);
3. gates, Eq.(1) (review page, paper sec.2) and q/k L2 normalisation;
4. the delta-rule recurrence, Eq.(2) (review page, paper sec.1), then the
   NVFP4 out_proj; optionally through the output gate of reading O1.

Every function states the reading it follows where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

FORM_PAGES = 0
FORM_STANDARD = 1


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (no fast-math, no FMA contraction)."""
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        subprocess.check_call([
            "gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
            "-shared", "-fPIC", src, "-o", _LIB_PATH, "-lm"])
    return _LIB_PATH


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i64, i32, f32, f64, u8 = ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_double, ctypes.c_uint8
        lib.orc_e2m1_decode.argtypes = [u8]; lib.orc_e2m1_decode.restype = f64
        lib.orc_e2m1_encode.argtypes = [f32]; lib.orc_e2m1_encode.restype = u8
        lib.orc_e4m3_decode.argtypes = [u8]; lib.orc_e4m3_decode.restype = f64
        lib.orc_e4m3_encode.argtypes = [f32]; lib.orc_e4m3_encode.restype = u8
        lib.orc_global_scale.argtypes = [P, i64]; lib.orc_global_scale.restype = f32
        lib.orc_quantize.argtypes = [P, i64, i64, f32, P, P]; lib.orc_quantize.restype = None
        lib.orc_dequantize.argtypes = [P, P, f32, i64, i64, P]; lib.orc_dequantize.restype = None
        lib.orc_sf_linear_to_mma.argtypes = [P, i64, i64, P]; lib.orc_sf_linear_to_mma.restype = None
        lib.orc_gemm_nt.argtypes = [P, P, i64, i64, i64, P]; lib.orc_gemm_nt.restype = None
        lib.orc_softplus.argtypes = [f64]; lib.orc_softplus.restype = f64
        lib.orc_output_gate.argtypes = [P, P, P, i64, i32, i32, f64, P]
        lib.orc_output_gate.restype = None
        lib.orc_short_conv.argtypes = [P, i64, i32, i64, i32, i32, P, P, P, P, i32]
        lib.orc_short_conv.restype = None
        lib.orc_gates.argtypes = [P, P, P, P, i64, i32, P, P]; lib.orc_gates.restype = None
        lib.orc_l2norm.argtypes = [P, i64, i32, f64]; lib.orc_l2norm.restype = None
        lib.orc_scan.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32, i32, f64, i32, P, P, P]
        lib.orc_scan.restype = None
        lib.orc_scan_chunked.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32, i32, f64, i32, i32,
                                         P, P, P]
        lib.orc_scan_chunked.restype = None
        lib.orc_scan_transition.argtypes = [P, P, P, P, i32, i64, i32, i32, i32, f64, i32, P, P]
        lib.orc_scan_transition.restype = None
        lib.orc_num_threads.argtypes = []; lib.orc_num_threads.restype = i32
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_L().orc_num_threads())


# ---------------------------------------------------------------- formats --
def e2m1_decode(code: int) -> float:
    return float(_L().orc_e2m1_decode(int(code)))


def e2m1_encode(y: float) -> int:
    return int(_L().orc_e2m1_encode(float(y)))


def e4m3_decode(b: int) -> float:
    return float(_L().orc_e4m3_decode(int(b)))


def e4m3_encode(s: float) -> int:
    return int(_L().orc_e4m3_encode(float(s)))


# -------------------------------------------------------------- quantiser --
def global_scale(x: np.ndarray) -> np.float32:
    """S = fl32(amax/2688), or 1 when amax < 2^-100 (reading Q1)."""
    x = _c(x, np.float32)
    return np.float32(_L().orc_global_scale(_p(x), x.size))


def quantize(x: np.ndarray, S: float | None = None):
    """NVFP4-quantise a float32 matrix [rows x cols] (cols % 16 == 0).

    Returns (codes uint8 [rows, cols/2], sf uint8 [rows, cols/16] linear, S).
    ``S`` given = use that global scale (harmonised weights); else computed
    from the tensor's amax.
    """
    x = _c(x, np.float32)
    rows, cols = x.shape
    assert cols % 16 == 0
    if S is None:
        S = global_scale(x)
    S = np.float32(S)
    codes = np.zeros((rows, cols // 2), np.uint8)
    sf = np.zeros((rows, cols // 16), np.uint8)
    _L().orc_quantize(_p(x), rows, cols, float(S), _p(codes), _p(sf))
    return codes, sf, S


def dequantize(codes: np.ndarray, sf: np.ndarray, S: float) -> np.ndarray:
    codes = _c(codes, np.uint8)
    sf = _c(sf, np.uint8)
    rows = codes.shape[0]
    cols = codes.shape[1] * 2
    out = np.empty((rows, cols), np.float64)
    _L().orc_dequantize(_p(codes), _p(sf), float(np.float32(S)), rows, cols, _p(out))
    return out


def sf_linear_to_mma(sf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Permute linear block scales into the tensor-core atom layout (rows
    padded to a multiple of 128 with zero bytes).  Returns a flat uint8 array."""
    sf = _c(sf, np.uint8)
    prow = (rows + 127) // 128 * 128
    out = np.empty(prow * (cols // 16), np.uint8)
    _L().orc_sf_linear_to_mma(_p(sf), rows, cols, _p(out))
    return out


# -------------------------------------------------------------------- GEMM --
def gemm_nt(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """C = A @ B^T in float64 (triple loop in C)."""
    A = _c(A, np.float64)
    B = _c(B, np.float64)
    M, K = A.shape
    N = B.shape[0]
    C = np.empty((M, N), np.float64)
    _L().orc_gemm_nt(_p(A), _p(B), M, N, K, _p(C))
    return C


def w4a4_gemm(Aq, Bq) -> np.ndarray:
    """Block-scaled FP4 GEMM reference: dequantise both operands exactly, then
    float64 C = A_hat @ B_hat^T (the product of S_A S_B and the block-scaled
    sums)."""
    A = dequantize(*Aq)
    B = dequantize(*Bq)
    return gemm_nt(A, B)


# -------------------------------------------------------------------- gates --
def softplus(u: float) -> float:
    return float(_L().orc_softplus(float(u)))


def gates(a: np.ndarray, b: np.ndarray, A_log: np.ndarray, dt_bias: np.ndarray):
    """Eq.(1): g = -exp(A_log) softplus(a + dt_bias), alpha = e^g, beta = sigmoid(b).
    a, b: [n, Hv].  Returns (g, beta) float64."""
    a = _c(a, np.float64)
    b = _c(b, np.float64)
    n, Hv = a.shape
    g = np.empty_like(a)
    beta = np.empty_like(a)
    _L().orc_gates(_p(a), _p(b), _p(_c(A_log, np.float64)), _p(_c(dt_bias, np.float64)), n, Hv,
                   _p(g), _p(beta))
    return g, beta


def l2norm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(sum x^2 + eps) along the last axis (reading G2)."""
    y = np.array(x, dtype=np.float64, order="C", copy=True)
    D = y.shape[-1]
    _L().orc_l2norm(_p(y), y.size // D, D, eps)
    return y


def output_gate(o: np.ndarray, z: np.ndarray, w: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """Optional output gate (reading O1 in oracle.c): per token and value head,
    o / sqrt(mean(o^2) + eps) * w * SiLU(z).  o, z: [..., Hv, V] (any leading
    shape); w: [V].  Returns float64 of o's shape."""
    o64 = _c(o, np.float64)
    z64 = _c(z, np.float64).reshape(o64.shape)
    V = o64.shape[-1]
    Hv = o64.shape[-2]
    out = np.empty_like(o64)
    _L().orc_output_gate(_p(o64), _p(z64), _p(_c(w, np.float64)), o64.size // (Hv * V), Hv, V, float(eps), _p(out))
    return out


def short_conv(x: np.ndarray, w: np.ndarray, B: int, T: int, state_in=None, silu: bool = True,
               return_state: bool = False):
    """Optional short causal convolution (reading C1 in oracle.c).  x: [B*T, C]
    (a column slice is fine); w: [C, W]; state_in: [B, C, W-1] or None.
    Returns out [B*T, C] float64 (and the new state [B, C, W-1])."""
    x64 = _c(x, np.float64)
    C, W = w.shape
    assert x64.shape == (B * T, C)
    out = np.empty((B * T, C), np.float64)
    st_out = np.empty((B, C, W - 1), np.float64) if return_state else None
    st_in = None if state_in is None else _c(state_in, np.float64)
    _L().orc_short_conv(_p(x64), C, B, T, C, W, _p(_c(w, np.float64)), None if st_in is None else _p(st_in),
                        None if st_out is None else _p(st_out), _p(out), 1 if silu else 0)
    return (out, st_out) if return_state else out


# --------------------------------------------------------------------- scan --
def scan(q, k, v, g, beta, scale=None, form=FORM_PAGES, S0=None):
    """Eq.(2) token by token.  q, k: [B,T,Hk,K]; v: [B,T,Hv,V]; g, beta: [B,T,Hv];
    S0: [B,Hv,K,V] or None.  Returns (o [B,T,Hv,V], S [B,Hv,K,V])."""
    q, k, v = _c(q, np.float64), _c(k, np.float64), _c(v, np.float64)
    g, beta = _c(g, np.float64), _c(beta, np.float64)
    B, T, Hk, K = q.shape
    Hv, V = v.shape[2], v.shape[3]
    if scale is None:
        scale = 1.0 / np.sqrt(K)
    S = np.empty((B, Hv, K, V), np.float64)
    o = np.empty((B, T, Hv, V), np.float64)
    s0 = None if S0 is None else _c(S0, np.float64)
    _L().orc_scan(_p(q), _p(k), _p(v), _p(g), _p(beta), B, T, Hk, Hv, K, V, float(scale), int(form),
                  None if s0 is None else _p(s0), _p(S), _p(o))
    return o, S


def scan_chunked(q, k, v, g, beta, chunk=64, scale=None, form=FORM_PAGES, S0=None):
    """Chunked restatement of Eq.(2) (pins the GPU kernel's derivation)."""
    q, k, v = _c(q, np.float64), _c(k, np.float64), _c(v, np.float64)
    g, beta = _c(g, np.float64), _c(beta, np.float64)
    B, T, Hk, K = q.shape
    Hv, V = v.shape[2], v.shape[3]
    if scale is None:
        scale = 1.0 / np.sqrt(K)
    S = np.empty((B, Hv, K, V), np.float64)
    o = np.empty((B, T, Hv, V), np.float64)
    s0 = None if S0 is None else _c(S0, np.float64)
    _L().orc_scan_chunked(_p(q), _p(k), _p(v), _p(g), _p(beta), B, T, Hk, Hv, K, V, float(scale),
                          int(form), int(chunk), None if s0 is None else _p(s0), _p(S), _p(o))
    return o, S


# ----------------------------------------------------------- state passing --
def scan_transition(q, k, g, beta, scale=None, form=FORM_PAGES):
    """Reading P1: the span's state map P = A_T...A_1 (A_t = a_t I - b_t k_t k_t^T,
    or a_t (I - b_t k_t k_t^T) in the STANDARD form) and the query map
    m_t = scale P_t^T q_t, formed token by token from the product itself.
    q, k: [B,T,Hk,K]; g, beta: [B,T,Hv].  Returns (P [B,Hv,K,K], m [B,T,Hv,K]).
    A span started from S_in then ends in P S_in + S_loc and its outputs gain
    S_in^T m_t (Eq.(2) is affine in the state; review page, background)."""
    q, k = _c(q, np.float64), _c(k, np.float64)
    g, beta = _c(g, np.float64), _c(beta, np.float64)
    B, T, Hk, K = q.shape
    Hv = g.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(K)
    P = np.empty((B, Hv, K, K), np.float64)
    m = np.empty((B, T, Hv, K), np.float64)
    _L().orc_scan_transition(_p(q), _p(k), _p(g), _p(beta), B, T, Hk, Hv, K, float(scale), int(form), _p(P), _p(m))
    return P, m


def state_combine(P, S_loc, S_in):
    """State at the end of a span that started from S_in: P S_in + S_loc, per
    (sequence, value head).  P: [...,K,K]; S_loc, S_in: [...,K,V]."""
    return np.matmul(np.asarray(P, np.float64), np.asarray(S_in, np.float64)) + np.asarray(S_loc, np.float64)


def output_correct(o_loc, m, S_in):
    """Outputs of a span that started from S_in, given its zero-start outputs
    o_loc [B,T,Hv,V] and query map m [B,T,Hv,K]: o_t = o_loc_t + S_in^T m_t,
    S_in [B,Hv,K,V]."""
    return np.asarray(o_loc, np.float64) + np.einsum("bthi,bhij->bthj", np.asarray(m, np.float64),
                                                     np.asarray(S_in, np.float64))


def scan_segmented(q, k, v, g, beta, bounds, scale=None, form=FORM_PAGES, S0=None):
    """Reading P1: the scan of each span [bounds[i], bounds[i+1]) from a zero
    state, the span maps, the spans' initial states by composing the maps in
    order from S0, then each span's outputs corrected by its initial state.
    Returns (o [B,T,Hv,V], S [B,Hv,K,V]) like scan()."""
    q, k, v = _c(q, np.float64), _c(k, np.float64), _c(v, np.float64)
    g, beta = _c(g, np.float64), _c(beta, np.float64)
    B, T, Hk, K = q.shape
    Hv, V = v.shape[2], v.shape[3]
    assert bounds[0] == 0 and bounds[-1] == T and all(a < b for a, b in zip(bounds, bounds[1:]))
    S = np.zeros((B, Hv, K, V)) if S0 is None else _c(S0, np.float64).copy()
    o = np.empty((B, T, Hv, V), np.float64)
    for a, b in zip(bounds, bounds[1:]):
        sl = slice(a, b)
        o_loc, S_loc = scan(q[:, sl], k[:, sl], v[:, sl], g[:, sl], beta[:, sl], scale=scale, form=form)
        P, m = scan_transition(q[:, sl], k[:, sl], g[:, sl], beta[:, sl], scale=scale, form=form)
        o[:, sl] = output_correct(o_loc, m, S)
        S = state_combine(P, S_loc, S)
    return o, S


# -------------------------------------------------------------------- layer --
def split_projection(P: np.ndarray, Hk: int, Hv: int, K: int, V: int):
    """Column slices of the fused projection, in the order q | k | v | z | a | b."""
    widths = [Hk * K, Hk * K, Hv * V, Hv * V, Hv, Hv]
    out, c = [], 0
    for w in widths:
        out.append(P[..., c:c + w])
        c += w
    return out


def layer_forward(x: np.ndarray, W_in_q, W_out_q, A_log, dt_bias, B: int, T: int, Hk: int, Hv: int,
                  K: int, V: int, form=FORM_PAGES, S0=None, stages: bool = False, W_in_deq=None,
                  W_out_deq=None, out_norm=None, conv_w=None, conv_state=None):
    """The four steps composed.  x: float32 [B*T, H] (bf16 values);
    W_in_q, W_out_q: (codes, sf_linear, S) of the fused in_proj [N_in, H] and
    out_proj [H, Hv*V] (or their dequantised float64 matrices in W_in_deq /
    W_out_deq, to skip re-dequantising fixed weights).  With ``out_norm`` (the
    weight w of V entries) the output gate of reading O1 is applied to o before
    out_proj.  With ``conv_w`` ([2 Hk K + Hv V, W]) the q|k|v columns of the
    projection first pass through the short convolution of reading C1, with
    ``conv_state`` ([B, C, W-1] or None) as the carried inputs.  Returns y
    [B*T, H] float64 and the final state (and every intermediate, with the new
    convolution state, when ``stages``)."""
    xq = quantize(x)                                            # step 1
    if W_in_deq is None:
        W_in_deq = dequantize(*W_in_q)
    if W_out_deq is None:
        W_out_deq = dequantize(*W_out_q)
    P = gemm_nt(dequantize(*xq), W_in_deq)                      # step 2
    conv_state_out = None
    Pc = P
    if conv_w is not None:                                      # optional short convolution
        C = 2 * Hk * K + Hv * V
        Pc = P.copy()
        Pc[:, :C], conv_state_out = short_conv(P[:, :C], conv_w, B, T, state_in=conv_state, return_state=True)
    q, k, v, _, _, _ = split_projection(Pc, Hk, Hv, K, V)
    _, _, _, z, a, b = split_projection(P, Hk, Hv, K, V)
    g, beta = gates(a, b, A_log, dt_bias)                       # step 3
    qh = l2norm(q.reshape(B, T, Hk, K))
    kh = l2norm(k.reshape(B, T, Hk, K))
    o, S = scan(qh, kh, v.reshape(B, T, Hv, V), g.reshape(B, T, Hv), beta.reshape(B, T, Hv),
                form=form, S0=S0)                               # step 4
    o2 = o.reshape(B * T, Hv * V).astype(np.float32)            # the out_proj reads fp32 o
    G = None
    if out_norm is not None:                                    # optional output gate
        G = output_gate(o2.reshape(B * T, Hv, V), z.reshape(B * T, Hv, V), out_norm)
        o2 = G.reshape(B * T, Hv * V).astype(np.float32)
    oq = quantize(o2)
    y = gemm_nt(dequantize(*oq), W_out_deq)
    if stages:
        return dict(xq=xq, P=P, Pc=Pc, conv_state=conv_state_out, g=g, beta=beta, q_hat=qh, k_hat=kh, o=o, S=S,
                    G=G, oq=oq, y=y)
    return y, S
