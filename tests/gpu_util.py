"""Helpers shared by the GPU parity tests (marshalling only, no arithmetic of
the method)."""
import numpy as np
import torch

import nvfp4_w4a4_gated_b200 as nv
import oracle


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def upload_oracle_nvfp4(q, rows, cols, dev="cuda"):
    """Oracle quantisation (codes, linear sf, S) -> device NVFP4Matrix (scales
    permuted into the atom layout by the oracle's own permutation)."""
    codes, sf, S = q
    m = nv.NVFP4Matrix.empty(rows, cols, dev)
    m.codes.copy_(torch.from_numpy(np.ascontiguousarray(codes)))
    m.sf.copy_(torch.from_numpy(oracle.sf_linear_to_mma(sf, rows, cols)))
    m.scale.fill_(float(np.float32(S)))
    return m


def bf16_device(bits_u16, dev="cuda"):
    return torch.from_numpy(bits_u16.view(np.int16)).to(dev).view(torch.bfloat16)


def f32_device(x, dev="cuda"):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dev)
