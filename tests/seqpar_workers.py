"""Rank bodies for the multi-process CPU tests of the sequence-parallel scan
(run under torch.multiprocessing.spawn with the gloo backend).  The span
steps are the oracle's, on float64 CPU tensors; what runs under test is the
host logic of nvfp4_w4a4_gated_b200.seqpar: rank order, the all-gather, the
composition of the maps and the corrections."""
import os

import numpy as np
import torch
import torch.distributed as dist

import gdn_synth
import oracle


class OracleSpanOps:
    """gdn_scan_span / gdn_state_combine / gdn_scan_correct restated with the
    oracle, in the binding's tensor shapes."""

    def local(self, q, k, v, g, beta, B, T, dims, scale, form):
        Hk, Hv, K, V = dims.Hk, dims.Hv, dims.K, dims.V
        qa, ka = q.numpy().reshape(B, T, Hk, K), k.numpy().reshape(B, T, Hk, K)
        ga, ba = g.numpy().reshape(B, T, Hv), beta.numpy().reshape(B, T, Hv)
        o, S = oracle.scan(qa, ka, v.numpy()[:, :Hv * V].reshape(B, T, Hv, V), ga, ba, scale=scale, form=form)
        P, m = oracle.scan_transition(qa, ka, ga, ba, scale=scale, form=form)
        return (torch.from_numpy(o.reshape(B * T, Hv, V)), torch.from_numpy(S), torch.from_numpy(P),
                torch.from_numpy(m.reshape(B * T, Hv, K)))

    def combine(self, P, S_loc, S_in):
        """P [m, ...], S_loc [m, ...]: fold the maps in order."""
        S = None if S_in is None else S_in.numpy()
        for j in range(P.shape[0]):
            S = S_loc[j].numpy().copy() if S is None else oracle.state_combine(P[j].numpy(), S_loc[j].numpy(), S)
        return torch.from_numpy(S)

    def correct(self, qmap, S_in, o, B, T):
        Hv, K, V = S_in.shape[1], S_in.shape[2], S_in.shape[3]
        out = oracle.output_correct(o.numpy().reshape(B, T, Hv, V), qmap.numpy().reshape(B, T, Hv, K), S_in.numpy())
        return torch.from_numpy(out.reshape(B * T, Hv, V))


def problem(form):
    """One seeded problem shared by every rank: 2 sequences of 90 tokens."""
    from nvfp4_w4a4_gated_b200 import GdnDims
    B, T, Hk, Hv, K, V = 2, 90, 2, 4, 8, 6
    q, k, v, g, beta = gdn_synth.scan_inputs(300, B, T, Hk, Hv, K, V, alpha_lo=0.7)
    S0 = gdn_synth.gaussian(301, (B, Hv, K, V)).astype(np.float64)
    return GdnDims(Hk, Hv, K, V), (q, k, v, g, beta), S0


def span_tensors(arrs, a, e, dims):
    """This rank's tokens [a, e) of every sequence, in the binding's shapes."""
    q, k, v, g, beta = (x[:, a:e].astype(np.float64) for x in arrs)
    B, T = q.shape[0], e - a
    t = lambda x, *shape: torch.from_numpy(np.ascontiguousarray(x).reshape(*shape))
    return (t(q, B * T, dims.Hk, dims.K), t(k, B * T, dims.Hk, dims.K), t(v, B * T, dims.Hv * dims.V),
            t(g, B * T, dims.Hv), t(beta, B * T, dims.Hv))


def rank_main(rank, world, port, bounds, form, with_state, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from nvfp4_w4a4_gated_b200.seqpar import sequence_parallel_scan
        dims, arrs, S0 = problem(form)
        a, e = bounds[rank], bounds[rank + 1]
        q, k, v, g, beta = span_tensors(arrs, a, e, dims)
        B = q.shape[0] // (e - a)
        o, S_end = sequence_parallel_scan(q, k, v, g, beta, B, e - a, dims, scale=None, form=form,
                                          state_in=torch.from_numpy(S0) if with_state else None,
                                          ops=OracleSpanOps())
        o_ref, _ = oracle.scan(*arrs, form=form, S0=S0 if with_state else None)
        _, S_ref = oracle.scan(*(x[:, :e] for x in arrs), form=form, S0=S0 if with_state else None)
        o_ref = o_ref[:, a:e].reshape(B * (e - a), dims.Hv, dims.V)
        err_o = float(np.max(np.abs(o.numpy() - o_ref)) / max(1.0, np.abs(o_ref).max()))
        err_S = float(np.max(np.abs(S_end.numpy() - S_ref)) / max(1.0, np.abs(S_ref).max()))
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{err_o} {err_S}\n")
    finally:
        dist.destroy_process_group()


def bench_rank_main(rank, world, port, out_dir):
    """bench.py's aggregation over gloo ranks: each rank reports its own times;
    all must come back with the maximum, and the throughput counts every
    rank's tokens over that time."""
    import importlib.util
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
        spec = importlib.util.spec_from_file_location("bench_agg", os.path.join(root, "bench.py"))
        b = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(b)
        mine = [10.0 + rank, 20.0 - rank]
        got = b.max_over_ranks(mine, torch.device("cpu"), True)
        tokens, value = b.job_throughput(world, 4096, 10, got[0])
        with open(os.path.join(out_dir, f"agg{rank}.txt"), "w") as f:
            f.write(f"{got[0]} {got[1]} {tokens} {value}\n")
    finally:
        dist.destroy_process_group()


# ------------------------------------------------------------ the layer --
class OracleLayerOps(OracleSpanOps):
    """The layer's other steps (quantiser modes, GEMM, gates) restated with the
    oracle, on CPU tensors, for nvfp4_w4a4_gated_b200.seqpar.sequence_parallel_layer."""

    def amax_word(self, x):
        a = np.float32(np.max(np.abs(np.asarray(x.numpy(), dtype=np.float32))))
        return torch.from_numpy(np.array([a], dtype=np.float32).view(np.int32))

    def quantize_from_amax(self, x, word):
        amax = word.numpy().view(np.float32)
        S = oracle.global_scale(amax)          # the per-tensor scale of a tensor whose amax is this word
        return oracle.quantize(np.asarray(x.numpy(), dtype=np.float32), S=S)

    def gemm(self, a, b):
        return torch.from_numpy(oracle.w4a4_gemm(a, b))

    def gates(self, P, w):
        d = w.dims
        q, k, v, _, a, b = oracle.split_projection(P.numpy(), d.Hk, d.Hv, d.K, d.V)
        g, beta = oracle.gates(a, b, w.A_log, w.dt_bias)
        n = P.shape[0]
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
        return (t(oracle.l2norm(q.reshape(n, d.Hk, d.K))), t(oracle.l2norm(k.reshape(n, d.Hk, d.K))), t(v), t(g),
                t(beta))


class OracleLayer:
    """Weights of the layer test: the oracle's quantised in_proj / out_proj."""

    def __init__(self, dims, w_in, w_out, A_log, dt_bias):
        self.dims, self.w_in, self.w_out, self.A_log, self.dt_bias = dims, w_in, w_out, A_log, dt_bias


def layer_problem(form):
    """One seeded layer shared by every rank: 2 sequences of 90 tokens, hidden 64."""
    from nvfp4_w4a4_gated_b200 import GdnDims
    dims = GdnDims(2, 4, 16, 16)
    B, T, H = 2, 90, 64
    _, x = gdn_synth.activations(310, B * T, H, hot="fixed")
    W_in = gdn_synth.weights(311, dims.n_in, H)
    W_out = gdn_synth.weights(312, H, dims.Hv * dims.V)
    A_log, dt_bias = gdn_synth.gate_params(313, dims.Hv)
    S0 = gdn_synth.gaussian(314, (B, dims.Hv, dims.K, dims.V), std=0.5).astype(np.float64)
    w = OracleLayer(dims, oracle.quantize(W_in), oracle.quantize(W_out), A_log, dt_bias)
    return w, x, B, T, H, S0


def layer_rank_main(rank, world, port, bounds, form, with_state, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from nvfp4_w4a4_gated_b200.seqpar import sequence_parallel_layer
        w, x, B, T, H, S0 = layer_problem(form)
        d = w.dims
        a, e = bounds[rank], bounds[rank + 1]
        x_loc = np.ascontiguousarray(x.reshape(B, T, H)[:, a:e].reshape(B * (e - a), H))
        y, xq, oq, S_end = sequence_parallel_layer(w, torch.from_numpy(x_loc), B, e - a, form=form,
                                                   state_in=torch.from_numpy(S0) if with_state else None,
                                                   ops=OracleLayerOps())
        ref = oracle.layer_forward(x, w.w_in, w.w_out, w.A_log, w.dt_bias, B, T, d.Hk, d.Hv, d.K, d.V, form=form,
                                   S0=S0 if with_state else None, stages=True)
        rows = lambda m: np.ascontiguousarray(m.reshape(B, T, -1)[:, a:e].reshape(B * (e - a), -1))
        same_x = (np.array_equal(xq[0], rows(ref["xq"][0])) and np.array_equal(xq[1], rows(ref["xq"][1]))
                  and np.float32(xq[2]) == np.float32(ref["xq"][2]))
        same_o = (np.array_equal(oq[0], rows(ref["oq"][0])) and np.array_equal(oq[1], rows(ref["oq"][1]))
                  and np.float32(oq[2]) == np.float32(ref["oq"][2]))
        y_ref = rows(ref["y"])
        err_y = float(np.max(np.abs(y.numpy() - y_ref)) / np.abs(y_ref).max())
        err_S = 0.0
        if rank == world - 1:
            err_S = float(np.max(np.abs(S_end.numpy() - ref["S"])) / np.abs(ref["S"]).max())
        with open(os.path.join(out_dir, f"layer{rank}.txt"), "w") as f:
            f.write(f"{int(same_x)} {int(same_o)} {err_y} {err_S}\n")
    finally:
        dist.destroy_process_group()
