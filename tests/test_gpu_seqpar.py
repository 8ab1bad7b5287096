"""The sequence split along time on one GPU, through the C ABI.

  * gdn_segment_map (M, N of a segment) against the oracle's segment map, on the tensor-core path
    (bf16, d = 128) and the CUDA-core path (fp32, d = 64);
  * gdn_state_compose (M S + N and M^T S + N) against float64 arithmetic;
  * every segment of a split sequence processed in turn on one GPU with seqpar's scans (the
    exchange between ranks replaced by holding every segment's map): each segment's output and
    gradients, the final state and the gradient of h0 against one oracle call over the whole
    sequence.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_76_b200 import gdn, seqpar
from gated_delta_rule_76_b200.inputs import draw
from oracle import oracle
from parity import assert_parity, npf, to_cuda

pytestmark = pytest.mark.gpu


def gates(x):
    return dict(beta=x["beta"]) if "beta" in x else dict(b=x["b"], w=x["w"])


@pytest.mark.parametrize("d,dtype,apc,gpc", [(128, "bf16", True, True), (128, "bf16", False, False),
                                             (64, "f32", True, True)])
def test_segment_map_matches_oracle(d, dtype, apc, gpc):
    x = draw(2, 150, 1, 2, d, d, alpha_per_channel=apc, gates_per_channel=gpc, dtype=dtype,
             gate_dtype=dtype if gpc or apc else "f32", seed=91, has_h0=False)
    g = to_cuda(x)
    M, N = gdn.gdn_segment_map(g["q"], g["k"], g["v"], g["alpha"], **gates(g))
    torch.cuda.synchronize()
    M_ref, N_ref = oracle.segment_map(x["q"], x["k"], x["v"], x["alpha"], **gates(x))
    kind = "f32" if dtype == "f32" else "bf16"
    assert_parity(M, M_ref, kind, "M")
    assert_parity(N, N_ref, kind, "N")


@pytest.mark.parametrize("dk,dv,transpose", [(128, 128, False), (128, 128, True), (64, 128, False), (64, 64, True)])
def test_state_compose(dk, dv, transpose):
    gen = torch.Generator().manual_seed(92)
    M = torch.randn((3, 2, dk, dk), generator=gen)
    N = torch.randn((3, 2, dk, dv), generator=gen)
    S = torch.randn((3, 2, dk, dv), generator=gen)
    out = gdn.gdn_state_compose(M.cuda(), N.cuda(), S.cuda(), transpose=transpose)
    torch.cuda.synchronize()
    ref = oracle.compose(M.numpy(), N.numpy(), S.numpy(), transpose=transpose)
    assert_parity(out, ref, "f32", "compose")
    only_n = gdn.gdn_state_compose(M.cuda(), N.cuda(), None, transpose=transpose)
    assert torch.equal(only_n.cpu(), N)


@pytest.mark.parametrize("cuts", [[0, 100, 180, 256], [0, 64, 192, 256]])
def test_split_sequence_on_one_gpu(cuts):
    B, T, Hk, Hv, d = 2, 256, 1, 2, 128
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=True, gates_per_channel=True, dtype="bf16",
             gate_dtype="bf16", seed=93, has_h0=True, with_dout=True, with_dht=True)
    g = to_cuda(x)
    ops = seqpar.DeviceOps(out_f32=True)  # every segment in turn, on this GPU
    segs = [{k: g[k][:, lo:hi].contiguous() for k in ("q", "k", "v", "alpha", "b", "w", "dout")}
            for lo, hi in zip(cuts[:-1], cuts[1:])]
    maps = [ops.segment_map(s) for s in segs]
    Ms, Ns = [m for m, _ in maps], [n for _, n in maps]
    outs, s_ins, ht = [], [], None
    for r, s in enumerate(segs):
        s_in = seqpar.entering_state(Ms, Ns, g["h0"], r, ops)
        o, ht_local = ops.forward(s, s_in, 1.0)
        outs.append(o)
        s_ins.append(s_in)
        ht = seqpar.final_state(Ms, Ns, ht_local, r, ops)  # the same on every segment
    Gs = [ops.backward(s, s_ins[r], s["dout"], None, 1.0)["dh0"] for r, s in enumerate(segs)]
    grads = [ops.backward(s, s_ins[r], s["dout"], seqpar.leaving_grad(Ms, Gs, g["dht"], r, ops), 1.0)
             for r, s in enumerate(segs)]
    torch.cuda.synchronize()
    o_ref, ht_ref = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], **gates(x))
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], dout=x["dout"], dht=x["dht"], **gates(x))
    o_all = torch.cat(outs, dim=1)
    assert_parity(o_all, o_ref, "bf16", "o")
    assert_parity(ht, ht_ref, "bf16", "final state")
    for key in ("dq", "dk", "dv", "dalpha", "db", "dw"):
        assert_parity(torch.cat([gr[key] for gr in grads], dim=1), ref[key], "bf16", key)
    assert_parity(grads[0]["dh0"], ref["dh0"], "bf16", "dh0")
