"""Fast-forgetting gates: decays whose product over a chunk leaves the chunk kernels' range.

The chunk kernels carry the decay inside a chunk of 64 tokens as a ratio of running products of
alpha; below a chunk product of 2^-100 on some channel the factors overflow.  Those (sequence, head)
pairs are marked by the chunk kernels and recomputed by the exact sequential kernels.  Checked here
against the fp64 oracle (a plain sequential recurrence, which has no such range):
  * alpha near 0.1 (down to ~1e-3) on some pairs, the recipe's alpha on the others, in one call:
    forward outputs, final states and every gradient, on the tensor-core path (bf16, d = 128) and on
    the CUDA-core path (fp32 and bf16, d = 64), with an initial state, a final-state gradient, GQA
    and a ragged last chunk;
  * the training step through the forward cache (forward keeping it, backward reading it);
  * a chunk product of 1e-28 on every channel (inside the range: the chunk path itself);
  * the GQA layer core, forward and backward, with fast-forgetting scalar gates.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_76_b200 import gdn
from gated_delta_rule_76_b200.inputs import draw
from oracle import oracle
from parity import assert_parity, npf, to_cuda

pytestmark = pytest.mark.gpu


def mixed_inputs(B, T, Hk, Hv, d, apc, gpc, dtype, gdt, seed, strong_pairs, conv=False):
    """The recipe's inputs, with the decay of the listed (sequence, value head) pairs replaced by a
    fast-forgetting one (alpha = exp(-3 softplus(x)))."""
    kw = dict(alpha_per_channel=apc, gates_per_channel=gpc, dtype=dtype, gate_dtype=gdt, seed=seed,
              has_h0=not conv, with_dout=True, with_dht=not conv, conv=conv, swish_gate=conv)
    x = draw(B, T, Hk, Hv, d, d, **kw)
    fast = draw(B, T, Hk, Hv, d, d, decay_scale=3.0, **kw)["alpha"]
    for b, h in strong_pairs:
        x["alpha"][b, :, h] = fast[b, :, h]
    return x


def gates(x):
    return dict(beta=x["beta"]) if "beta" in x else dict(b=x["b"], w=x["w"])


CASES = [
    # tensor-core path: bf16, d = 128, channel gates (GDN-2) and scalar gates (GDN, fp32 gates)
    dict(d=128, apc=True, gpc=True, dtype="bf16", gdt="bf16"),
    dict(d=128, apc=False, gpc=False, dtype="bf16", gdt="f32"),
    # CUDA-core path: fp32 and bf16 tensors, d = 64
    dict(d=64, apc=True, gpc=True, dtype="f32", gdt="f32"),
    dict(d=64, apc=True, gpc=False, dtype="bf16", gdt="bf16"),
]


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"d{c['d']}-{c['dtype']}-{'ch' if c['apc'] else 'sc'}")
def test_fast_forgetting_pairs_forward_and_backward(c):
    B, T, Hk, Hv = 2, 200, 2, 4
    strong = [(0, 1), (0, 2)] + [(1, h) for h in range(Hv)]
    x = mixed_inputs(B, T, Hk, Hv, c["d"], c["apc"], c["gpc"], c["dtype"], c["gdt"], 61, strong)
    a = npf(x["alpha"])
    assert a[0, :, 1].min() < 0.01 and np.prod(a[0, :64, 1], axis=0).min() < 1e-40, "the pair must leave the range"
    g = to_cuda(x)
    kind = "f32" if c["dtype"] == "f32" else "bf16"
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], out_f32=True, **gates(g))
    grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], grad_o=g["dout"], grad_ht=g["dht"],
                              **gates(g))
    torch.cuda.synchronize()
    o_ref, ht_ref = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], **gates(x))
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], dout=x["dout"], dht=x["dht"], **gates(x))
    for b in range(B):
        for h in range(Hv):
            tag = f"({b},{h}){' fast' if (b, h) in strong else ''}"
            assert_parity(o[b, :, h], o_ref[b, :, h], kind, f"o {tag}")
            assert_parity(ht[b, h], ht_ref[b, h], kind, f"ht {tag}")
            for key in ["dv", "dalpha"] + (["db", "dw"] if c["gpc"] else ["dbeta"]):
                assert_parity(grads[key][b, :, h], ref[key][b, :, h], kind, f"{key} {tag}")
            assert_parity(grads["dh0"][b, h], ref["dh0"][b, h], kind, f"dh0 {tag}")
        for hk in range(Hk):
            assert_parity(grads["dq"][b, :, hk], ref["dq"][b, :, hk], kind, f"dq ({b},{hk})")
            assert_parity(grads["dk"][b, :, hk], ref["dk"][b, :, hk], kind, f"dk ({b},{hk})")


def test_training_step_through_the_cache_with_fast_forgetting():
    """The forward keeps its cache (whose entries for out-of-range pairs are not meaningful) and the
    backward reads it: the backward's own range check sends those pairs to the sequential path."""
    B, T, Hk, Hv, d = 2, 192, 2, 2, 128
    strong = [(0, 0), (1, 1)]
    x = mixed_inputs(B, T, Hk, Hv, d, True, True, "bf16", "bf16", 62, strong)
    g = to_cuda(x)
    cache = torch.empty(gdn.gdn_chunk_fwd_cache_size(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], **gates(g)),
                        dtype=torch.uint8, device="cuda")
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], out_f32=True, bwd_cache=cache,
                              **gates(g))
    grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], grad_o=g["dout"], fwd_cache=cache,
                              **gates(g))
    torch.cuda.synchronize()
    o_ref, ht_ref = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], **gates(x))
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], dout=x["dout"], **gates(x))
    assert_parity(o, o_ref, "bf16", "o")
    assert_parity(ht, ht_ref, "bf16", "ht")
    for key in ("dq", "dk", "dv", "dalpha", "db", "dw", "dh0"):
        assert_parity(grads[key], ref[key], "bf16", key)


def test_chunk_product_near_1e_28_stays_on_the_chunk_path():
    """alpha = 0.3652 on every channel: the product over a full chunk is ~1e-28, inside the range
    (2^-100 ~ 7.9e-31), so the chunk kernels compute it with their factors."""
    B, T, Hk, Hv, d = 1, 256, 1, 2, 128
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=True, gates_per_channel=True, dtype="bf16", gate_dtype="bf16",
             seed=63, has_h0=True, with_dout=True)
    x["alpha"] = torch.full_like(x["alpha"], 0.3652)
    prod = float(np.prod(npf(x["alpha"][0, :64, 0, 0])))
    assert 7.9e-31 < prod < 2e-28
    g = to_cuda(x)
    launches0 = gdn.kernel_launches()
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], out_f32=True, **gates(g))
    grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], grad_o=g["dout"], **gates(g))
    torch.cuda.synchronize()
    assert gdn.kernel_launches() > launches0
    o_ref, ht_ref = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], **gates(x))
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], dout=x["dout"], **gates(x))
    assert_parity(o, o_ref, "bf16", "o")
    assert_parity(ht, ht_ref, "bf16", "ht")
    for key in ("dq", "dk", "dv", "dalpha", "db", "dw", "dh0"):
        assert_parity(grads[key], ref[key], "bf16", key)


@pytest.mark.parametrize("cached", [False, True])
def test_layer_core_with_fast_forgetting_heads(cached):
    """The GQA layer core (conv + SiLU + L2, recurrence, swish gate) on its tensor-core form with
    fast-forgetting scalar decays on some value heads: forward and backward against the oracle."""
    B, T, Hk, Hv, d = 1, 160, 1, 4, 128
    strong = [(0, 1), (0, 3)]
    x = mixed_inputs(B, T, Hk, Hv, d, False, False, "bf16", "f32", 64, strong, conv=True)
    g = to_cuda(x)
    lin = (g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"])
    cache = None
    if cached:
        cache = torch.empty(gdn.gdn_layer_core_fwd_cache_size(*lin, beta=g["beta"]), dtype=torch.uint8, device="cuda")
    y, ht, _ = gdn.gdn_layer_core_fwd(*lin, beta=g["beta"], out_f32=True, bwd_cache=cache)
    got = gdn.gdn_layer_core_bwd(*lin, g["dout"], beta=g["beta"], fwd_cache=cache)
    torch.cuda.synchronize()
    y_ref, ht_ref = oracle.layer_core_fwd(x["q"], x["k"], x["v"], x["conv_w"], x["alpha"], x["beta"], x["z"])
    assert_parity(y, y_ref, "bf16", "y")
    assert_parity(ht, ht_ref, "bf16", "ht")
    ref = oracle.layer_core_bwd(npf(x["q"]), npf(x["k"]), npf(x["v"]), npf(x["conv_w"]), npf(x["alpha"]),
                                npf(x["z"]), npf(x["dout"]), beta=npf(x["beta"]))
    for key in ("dxq", "dxk", "dxv", "dz", "dalpha", "dbeta"):
        assert_parity(got[key], ref[key], "bf16", key)
    assert_parity(got["dconv_w"], ref["dconv_w"], "bf16", "dconv_w")
