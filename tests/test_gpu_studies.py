"""The mechanism studies through the CUDA kernels against the same studies
through the oracle's steps, on the tiny layer: every number of the three
tables within a few percent (the GPU path rounds products to TF32 and its
GEMM accumulates in float32; the studies report errors of several percent)."""
import numpy as np
import pytest

import gdn_synth
from nvfp4_w4a4_gated_b200 import GdnDims, studies
from study_oracle_backend import OracleBackend

pytestmark = pytest.mark.gpu


def _both(T, seed=50):
    sh = gdn_synth.TINY
    dims = GdnDims(sh.Hk, sh.Hv, sh.K, sh.V)
    W_in = gdn_synth.weights(seed, sh.n_in, sh.H)
    W_out = gdn_synth.weights(seed + 1, sh.H, sh.Hv * sh.V)
    A_log, dt_bias = gdn_synth.gate_params(seed + 2, sh.Hv)
    _, x = gdn_synth.activations(seed + 3, T, sh.H, hot="fixed")
    out = []
    for be in (studies.CudaBackend(), OracleBackend()):
        L = studies.StudyLayer.make(be, W_in, W_out, A_log, dt_bias, dims, sh.H)
        out.append((be, L, be.upload(x)))
    return out


def _close(a, b, rel=0.05, abs_=2e-3):
    return abs(a - b) <= rel * abs(b) + abs_


def test_sensitivity_gpu_matches_oracle(cuda_dev):
    (gb, gL, gx), (ob, oL, ox) = _both(128)
    g = studies.sensitivity(gb, gL, gx, 1, 128)
    o = studies.sensitivity(ob, oL, ox, 1, 128)
    for name, row in o["rows"].items():
        for key, val in row.items():
            assert _close(g["rows"][name][key], val), (name, key, g["rows"][name][key], val)
    for key in ("joint_y_rel", "joint_state_rel", "rss_y_rel"):
        assert _close(g[key], o[key]), (key, g[key], o[key])


def test_lockstep_and_gate_noise_gpu_match_oracle(cuda_dev):
    (gb, gL, gx), (ob, oL, ox) = _both(256)
    g = studies.lockstep(gb, gL, gx, 256, [64, 128, 256], n_perturbed=3)
    o = studies.lockstep(ob, oL, ox, 256, [64, 128, 256], n_perturbed=3)
    for cg, co in zip(g["checkpoints"], o["checkpoints"]):
        for key in ("relS_mean", "relS_max", "relS_w4a4"):
            assert _close(cg[key], co[key]), (cg["t"], key, cg[key], co[key])
    g = studies.gate_noise(gb, gL, gx, 256)
    o = studies.gate_noise(ob, oL, ox, 256)
    for k in g:
        assert _close(g[k]["state_rel"], o[k]["state_rel"]), (k, g[k], o[k])
