"""Gates given as logits: alpha = exp(-alpha_scale[h] softplus(x)), b, w, beta = sigmoid(x), applied by
every kernel where it reads a gate; the backward returns the gradients of the logits and of
alpha_scale.  Against the oracle (its gate functions in float64, then its recurrence and reverse
mode, then its chain rule):
  * the chunk forward and backward on the tensor-core path (channel gates: the GDN-2 case; scalar
    gates) and the CUDA-core path (fp32, d = 64), and with a large alpha_scale (fast forgetting:
    the sequential path);
  * the training step through the forward cache;
  * decode steps;
  * the GQA layer core (scalar gates: the layer's a and beta projections), forward and backward.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_76_b200 import gdn
from gated_delta_rule_76_b200.inputs import draw
from oracle import oracle
from parity import assert_parity, npf, to_cuda

pytestmark = pytest.mark.gpu


def with_logits(x, apc, gpc, gdt, seed, scale_range=(0.05, 0.3)):
    """Replace the drawn gates by seeded logits (cast once to the gate dtype) and draw alpha_scale."""
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if gdt == "bf16" else torch.float32
    lg = lambda t: torch.randn(t.shape, generator=g).to(dt)
    x = dict(x)
    x["alpha"] = lg(x["alpha"])
    if gpc:
        x["b"], x["w"] = lg(x["b"]), lg(x["w"])
    else:
        x["beta"] = lg(x["beta"])
    Hv = x["v"].shape[-2]
    lo, hi = scale_range
    x["alpha_scale"] = (lo + (hi - lo) * torch.rand(Hv, generator=g)).float()
    return x


def oracle_gates(x):
    lg = dict(x_b=x["b"], x_w=x["w"]) if "b" in x else dict(x_beta=x["beta"])
    al, b, w, beta = oracle.gates_from_logits(x["alpha"], x["alpha_scale"], **lg)
    return al, (dict(b=b, w=w) if "b" in x else dict(beta=beta))


def oracle_logit_grads(x, ref):
    if "b" in x:
        return oracle.logit_grads(x["alpha"], x["alpha_scale"], ref["dalpha"], x_b=x["b"], db=ref["db"],
                                  x_w=x["w"], dw=ref["dw"])
    return oracle.logit_grads(x["alpha"], x["alpha_scale"], ref["dalpha"], x_beta=x["beta"], dbeta=ref["dbeta"])


def gates(x):
    return dict(beta=x["beta"]) if "beta" in x else dict(b=x["b"], w=x["w"])


CASES = [
    dict(d=128, apc=True, gpc=True, dtype="bf16", gdt="bf16", fast=False),
    dict(d=128, apc=False, gpc=False, dtype="bf16", gdt="f32", fast=False),
    dict(d=64, apc=True, gpc=True, dtype="f32", gdt="f32", fast=False),
    dict(d=128, apc=True, gpc=True, dtype="bf16", gdt="bf16", fast=True),
]


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"d{c['d']}-{c['dtype']}-{'ch' if c['apc'] else 'sc'}"
                                                   f"{'-fast' if c['fast'] else ''}")
def test_chunk_forward_backward_from_logits(c):
    B, T, Hk, Hv = 2, 150, 1, 2
    x = draw(B, T, Hk, Hv, c["d"], c["d"], alpha_per_channel=c["apc"], gates_per_channel=c["gpc"],
             dtype=c["dtype"], gate_dtype=c["gdt"], seed=111, has_h0=True, with_dout=True)
    x = with_logits(x, c["apc"], c["gpc"], c["gdt"], 112, (2.0, 4.0) if c["fast"] else (0.05, 0.3))
    g = to_cuda(x)
    kw = dict(h0=g["h0"], alpha_scale=g["alpha_scale"], **gates(g))
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], out_f32=True, **kw)
    grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], grad_o=g["dout"], **kw)
    torch.cuda.synchronize()
    al, gk = oracle_gates(x)
    if c["fast"]:
        assert np.prod(al[0, :64, 0], axis=0).min() < 1e-31, "alpha_scale must push the pair out of the range"
    o_ref, ht_ref = oracle.fwd(x["q"], x["k"], x["v"], al, h0=x["h0"], **gk)
    ref = oracle.bwd(x["q"], x["k"], x["v"], al, h0=x["h0"], dout=x["dout"], **gk)
    lref = oracle_logit_grads(x, ref)
    kind = "f32" if c["dtype"] == "f32" else "bf16"
    assert_parity(o, o_ref, kind, "o")
    assert_parity(ht, ht_ref, kind, "ht")
    for key in ("dq", "dk", "dv", "dh0"):
        assert_parity(grads[key], ref[key], kind, key)
    for key in ["dalpha", "dalpha_scale"] + (["db", "dw"] if c["gpc"] else ["dbeta"]):
        assert_parity(grads[key], lref[key], kind, f"{key} (logit)")


def test_training_step_from_logits_through_the_cache():
    B, T, Hk, Hv, d = 2, 128, 2, 2, 128
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=True, gates_per_channel=True, dtype="bf16", gate_dtype="bf16",
             seed=113, has_h0=True, with_dout=True)
    x = with_logits(x, True, True, "bf16", 114)
    g = to_cuda(x)
    kw = dict(h0=g["h0"], alpha_scale=g["alpha_scale"], **gates(g))
    cache = torch.empty(gdn.gdn_chunk_fwd_cache_size(g["q"], g["k"], g["v"], g["alpha"], **kw), dtype=torch.uint8,
                        device="cuda")
    o, _ = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], out_f32=True, bwd_cache=cache, **kw)
    grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], grad_o=g["dout"], fwd_cache=cache, **kw)
    torch.cuda.synchronize()
    al, gk = oracle_gates(x)
    o_ref, _ = oracle.fwd(x["q"], x["k"], x["v"], al, h0=x["h0"], **gk)
    ref = oracle.bwd(x["q"], x["k"], x["v"], al, h0=x["h0"], dout=x["dout"], **gk)
    lref = oracle_logit_grads(x, ref)
    assert_parity(o, o_ref, "bf16", "o")
    for key in ("dq", "dk", "dv"):
        assert_parity(grads[key], ref[key], "bf16", key)
    for key in ("dalpha", "db", "dw", "dalpha_scale"):
        assert_parity(grads[key], lref[key], "bf16", f"{key} (logit)")


def test_decode_steps_from_logits():
    N, Hk, Hv, d, steps = 3, 1, 2, 128, 4
    x = draw(N, steps, Hk, Hv, d, d, alpha_per_channel=True, gates_per_channel=True, dtype="bf16", gate_dtype="bf16",
             seed=115, has_h0=True)
    x = with_logits(x, True, True, "bf16", 116)
    g = to_cuda(x)
    state = g["h0"].clone()
    ref_state = npf(x["h0"])
    al, gk = oracle_gates(x)
    for t in range(steps):
        tk = lambda src, key: src[key][:, t].contiguous()
        o = gdn.gdn_decode_step(state, tk(g, "q"), tk(g, "k"), tk(g, "v"), tk(g, "alpha"), b=tk(g, "b"),
                                w=tk(g, "w"), alpha_scale=g["alpha_scale"], out_f32=True)
        o_ref, ref_state = oracle.decode_step(ref_state, tk(x, "q"), tk(x, "k"), tk(x, "v"), al[:, t],
                                              b=gk["b"][:, t], w=gk["w"][:, t])
        assert_parity(o, o_ref, "bf16", f"o step {t}")
    assert_parity(state, ref_state, "bf16", "state")


@pytest.mark.parametrize("cached", [False, True])
def test_layer_core_from_logits(cached):
    B, T, Hk, Hv, d = 1, 140, 1, 4, 128
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=False, gates_per_channel=False, dtype="bf16", gate_dtype="f32",
             seed=117, has_h0=False, conv=True, swish_gate=True, with_dout=True)
    x = with_logits(x, False, False, "f32", 118)
    g = to_cuda(x)
    lin = (g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"])
    kw = dict(beta=g["beta"], alpha_scale=g["alpha_scale"])
    cache = None
    if cached:
        cache = torch.empty(gdn.gdn_layer_core_fwd_cache_size(*lin, beta=g["beta"]), dtype=torch.uint8, device="cuda")
    y, ht, _ = gdn.gdn_layer_core_fwd(*lin, out_f32=True, bwd_cache=cache, **kw)
    got = gdn.gdn_layer_core_bwd(*lin, g["dout"], fwd_cache=cache, **kw)
    torch.cuda.synchronize()
    al, gk = oracle_gates(x)
    y_ref, ht_ref = oracle.layer_core_fwd(x["q"], x["k"], x["v"], x["conv_w"], al, gk["beta"], x["z"])
    assert_parity(y, y_ref, "bf16", "y")
    assert_parity(ht, ht_ref, "bf16", "ht")
    ref = oracle.layer_core_bwd(npf(x["q"]), npf(x["k"]), npf(x["v"]), npf(x["conv_w"]), al, npf(x["z"]),
                                npf(x["dout"]), beta=gk["beta"])
    lref = oracle.logit_grads(x["alpha"], x["alpha_scale"], ref["dalpha"], x_beta=x["beta"], dbeta=ref["dbeta"])
    for key in ("dxq", "dxk", "dxv", "dz"):
        assert_parity(got[key], ref[key], "bf16", key)
    for key in ("dalpha", "dbeta", "dalpha_scale"):
        assert_parity(got[key], lref[key], "bf16", f"{key} (logit)")
