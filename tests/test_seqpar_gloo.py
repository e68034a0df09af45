"""The sequence-parallel scan's host logic on 2 and 3 CPU ranks (gloo): every
rank's outputs and end-of-span state must equal the whole-sequence recurrence
of the oracle.  The span steps are the oracle's (see seqpar_workers)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import oracle
import seqpar_workers


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("bounds,form,with_state", [
    ([0, 45, 90], oracle.FORM_PAGES, False),
    ([0, 45, 90], oracle.FORM_STANDARD, True),
    ([0, 10, 11, 90], oracle.FORM_STANDARD, True),     # a one-token span in the middle
    ([0, 64, 70, 90], oracle.FORM_PAGES, True),
])
def test_sequence_parallel_scan_on_gloo_ranks(tmp_path, bounds, form, with_state):
    world = len(bounds) - 1
    mp.spawn(seqpar_workers.rank_main, args=(world, _free_port(), bounds, form, with_state, str(tmp_path)),
             nprocs=world, join=True)
    for r in range(world):
        err_o, err_S = map(float, open(os.path.join(tmp_path, f"rank{r}.txt")).read().split())
        assert err_o < 1e-12 and err_S < 1e-12, (r, err_o, err_S)


def test_single_process_path_needs_no_process_group():
    """World of one (no process group): the scan of the whole span, joined
    with the initial state."""
    import numpy as np
    import torch
    from nvfp4_w4a4_gated_b200.seqpar import sequence_parallel_scan, segmented_scan
    dims, arrs, S0 = seqpar_workers.problem(oracle.FORM_PAGES)
    ops = seqpar_workers.OracleSpanOps()
    q, k, v, g, beta = seqpar_workers.span_tensors(arrs, 0, 90, dims)
    o, S = sequence_parallel_scan(q, k, v, g, beta, 2, 90, dims, state_in=torch.from_numpy(S0), ops=ops)
    o_ref, S_ref = oracle.scan(*arrs, S0=S0)
    assert np.allclose(o.numpy(), o_ref.reshape(180, dims.Hv, dims.V), atol=1e-12)
    assert np.allclose(S.numpy(), S_ref, atol=1e-12)
    spans = [seqpar_workers.span_tensors(arrs, a, e, dims) + (e - a,) for a, e in [(0, 30), (30, 31), (31, 90)]]
    outs, S2 = segmented_scan(spans, 2, dims, state_in=torch.from_numpy(S0), ops=ops)
    got = np.concatenate([o.numpy().reshape(2, -1, dims.Hv, dims.V) for o in outs], axis=1)
    assert np.allclose(got, o_ref, atol=1e-12) and np.allclose(S2.numpy(), S_ref, atol=1e-12)


def test_bench_aggregation_on_gloo_ranks(tmp_path):
    """bench.py under N ranks: the max over ranks of each timing and the
    whole-job throughput (all ranks' tokens over the slowest time)."""
    world = 2
    mp.spawn(seqpar_workers.bench_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        t0, t1, tokens, value = map(float, open(os.path.join(tmp_path, f"agg{r}.txt")).read().split())
        assert (t0, t1) == (11.0, 20.0)
        assert tokens == 2 * 4096 * 10 and abs(value - tokens / 0.011) < 1e-6 * value


@pytest.mark.parametrize("bounds,form,with_state", [
    ([0, 45, 90], oracle.FORM_PAGES, False),
    ([0, 10, 11, 90], oracle.FORM_STANDARD, True),     # a one-token span in the middle
    ([0, 30, 64, 90], oracle.FORM_PAGES, True),
])
def test_sequence_parallel_layer_on_gloo_ranks(tmp_path, bounds, form, with_state):
    """The whole layer with its tokens split across 2 and 3 CPU ranks (the
    steps are the oracle's): each rank's quantised x and o are the rows of the
    whole tensors' quantisation, bit for bit (one scale per tensor, from a max
    all-reduce of the ranks' amax words), and its y rows and the last rank's
    state equal the oracle's whole-sequence layer."""
    world = len(bounds) - 1
    mp.spawn(seqpar_workers.layer_rank_main, args=(world, _free_port(), bounds, form, with_state, str(tmp_path)),
             nprocs=world, join=True)
    for r in range(world):
        same_x, same_o, err_y, err_S = open(os.path.join(tmp_path, f"layer{r}.txt")).read().split()
        assert same_x == "1" and same_o == "1", (r, same_x, same_o)
        assert float(err_y) < 1e-12 and float(err_S) < 1e-12, (r, err_y, err_S)
