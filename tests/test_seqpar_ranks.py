"""Host logic of the sequence split along time (gated_delta_rule_76_b200/seqpar.py) on CPU.

Two and three ranks over gloo (127.0.0.1) each hold one segment of every sequence.  The oracle
stands in for the library's kernels (segment map, composition, forward, backward), so what is
tested is the exchange: the all-gather of the maps, the exclusive scan that gives each rank the
state entering its segment, and the reverse scan that carries the final state's gradient back.
Every rank's output and gradients must equal one sequential oracle call over the whole sequence.
"""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(T):
    sys.path.insert(0, ROOT)
    from gated_delta_rule_76_b200.inputs import draw
    x = draw(2, T, 1, 2, 8, 8, alpha_per_channel=True, gates_per_channel=True, dtype="f32", seed=81,
             has_h0=True, with_dout=True, with_dht=True)
    return {k: v.double() for k, v in x.items()}


class OracleOps:
    """seqpar's operations on the CPU oracle (float64 torch tensors in, out)."""

    def __init__(self):
        import torch
        from oracle import oracle
        self.o, self.torch = oracle, torch

    def _t(self, a):
        return self.torch.from_numpy(np.ascontiguousarray(a))

    def segment_map(self, x):
        M, N = self.o.segment_map(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"])
        return self._t(M), self._t(N)

    def compose(self, M, N, S, transpose=False):
        return self._t(self.o.compose(M, N, S, transpose=transpose))

    def forward(self, x, h0, scale):
        o, ht = self.o.fwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=h0, scale=scale)
        return self._t(o), self._t(ht)

    def backward(self, x, h0, grad_o, grad_ht, scale):
        g = self.o.bwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=h0, scale=scale,
                       dout=grad_o, dht=grad_ht)
        return {k: self._t(v) for k, v in g.items()}


def _rank(rank, world, port, T, cuts, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import torch.distributed as dist
    from gated_delta_rule_76_b200 import seqpar
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    x = _inputs(T)
    lo, hi = cuts[rank], cuts[rank + 1]
    seg = {k: x[k][:, lo:hi].contiguous() for k in ("q", "k", "v", "alpha", "b", "w", "dout")}
    ops = OracleOps()
    f = seqpar.forward(seg, h0=x["h0"], scale=0.7, ops=ops)
    g = seqpar.backward(seg, f, seg["dout"], grad_ht=x["dht"], scale=0.7, ops=ops)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, f["o"].numpy(), f["ht"].numpy(), {k: v.numpy() for k, v in g.items()}))


@pytest.mark.parametrize("cuts", [[0, 40, 97], [0, 30, 64, 97]])
def test_ranks_reproduce_one_sequential_call(cuts):
    T, world = 97, len(cuts) - 1
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, T, cuts, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((out.get(timeout=180) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle import oracle
    x = _inputs(T)
    o_ref, ht_ref = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"], scale=0.7)
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"], scale=0.7,
                     dout=x["dout"], dht=x["dht"])
    rel = lambda a, b: float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))
    for rank, o, ht, g in res:
        lo, hi = cuts[rank], cuts[rank + 1]
        assert rel(o, o_ref[:, lo:hi]) < 1e-12, f"o, rank {rank}"
        assert rel(ht, ht_ref) < 1e-12, f"final state, rank {rank}"
        for key in ("dq", "dk", "dv", "dalpha", "db", "dw"):
            assert rel(g[key], ref[key][:, lo:hi]) < 1e-10, f"{key}, rank {rank}"
    assert rel(res[0][3]["dh0"], ref["dh0"]) < 1e-10, "gradient of h0 (rank 0)"
