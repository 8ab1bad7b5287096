"""The GQA layer core with its output norm before the gate, y = RMSNorm(o) * norm_w * swish(z),
against the oracle, forward and backward (every gradient, the norm weights' included):
  * the tensor-core form (bf16, d = 128, scalar gates), with and without the forward's cache; the
    norm is fused in the chunk forward's epilogue;
  * the CUDA-core form (channel gates; d = 64 fp32), where o is normalised row by row after the
    recurrence;
  * fast-forgetting heads on the tensor-core form (the sequential kernel's own norm).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_76_b200 import gdn
from gated_delta_rule_76_b200.inputs import draw
from oracle import oracle
from parity import assert_parity, npf, to_cuda

pytestmark = pytest.mark.gpu


def inputs(B, T, Hk, Hv, d, apc, gpc, dtype, gdt, seed, fast_heads=()):
    kw = dict(alpha_per_channel=apc, gates_per_channel=gpc, dtype=dtype, gate_dtype=gdt, seed=seed, has_h0=False,
              conv=True, swish_gate=True, with_dout=True)
    x = draw(B, T, Hk, Hv, d, d, **kw)
    if fast_heads:
        fast = draw(B, T, Hk, Hv, d, d, decay_scale=3.0, **kw)["alpha"]
        for h in fast_heads:
            x["alpha"][:, :, h] = fast[:, :, h]
    g = torch.Generator().manual_seed(seed)
    x["norm_w"] = (1.0 + 0.3 * torch.randn(d, generator=g)).to(x["q"].dtype)
    return x


def gates(x):
    return dict(beta=x["beta"]) if "beta" in x else dict(b=x["b"], w=x["w"])


def oracle_fwd(x):
    if "beta" in x:
        return oracle.layer_core_fwd(x["q"], x["k"], x["v"], x["conv_w"], x["alpha"], x["beta"], x["z"],
                                     norm_w=x["norm_w"])
    B, T, Hk, d = x["q"].shape
    Hv = x["v"].shape[2]
    cq = Hk * d
    w = npf(x["conv_w"])
    q, _ = oracle.conv_silu(npf(x["q"]).reshape(B, T, cq), w[:cq])
    k, _ = oracle.conv_silu(npf(x["k"]).reshape(B, T, cq), w[cq:2 * cq])
    v, _ = oracle.conv_silu(npf(x["v"]).reshape(B, T, Hv * d), w[2 * cq:])
    o, ht = oracle.fwd(oracle.l2norm(q.reshape(B, T, Hk, d)), oracle.l2norm(k.reshape(B, T, Hk, d)),
                       v.reshape(B, T, Hv, d), x["alpha"], **gates(x))
    return oracle.gated_rmsnorm(o, x["z"], x["norm_w"]), ht


CASES = [
    dict(d=128, apc=False, gpc=False, dtype="bf16", gdt="f32", cached=False, fast=()),
    dict(d=128, apc=False, gpc=False, dtype="bf16", gdt="f32", cached=True, fast=()),
    dict(d=128, apc=False, gpc=False, dtype="bf16", gdt="f32", cached=False, fast=(1,)),
    dict(d=128, apc=True, gpc=True, dtype="bf16", gdt="bf16", cached=False, fast=()),
    dict(d=64, apc=False, gpc=False, dtype="f32", gdt="f32", cached=False, fast=()),
]


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"d{c['d']}-{c['dtype']}-{'ch' if c['apc'] else 'sc'}"
                                                   f"{'-cache' if c['cached'] else ''}{'-fast' if c['fast'] else ''}")
def test_layer_core_with_output_norm(c):
    B, T, Hk, Hv = 2, 150, 1, 4
    x = inputs(B, T, Hk, Hv, c["d"], c["apc"], c["gpc"], c["dtype"], c["gdt"], 101, c["fast"])
    g = to_cuda(x)
    lin = (g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"])
    cache = None
    if c["cached"]:
        cache = torch.empty(gdn.gdn_layer_core_fwd_cache_size(*lin, norm_w=g["norm_w"], **gates(g)),
                            dtype=torch.uint8, device="cuda")
    y, ht, _ = gdn.gdn_layer_core_fwd(*lin, norm_w=g["norm_w"], out_f32=True, bwd_cache=cache, **gates(g))
    got = gdn.gdn_layer_core_bwd(*lin, g["dout"], norm_w=g["norm_w"], fwd_cache=cache, **gates(g))
    torch.cuda.synchronize()
    kind = "f32" if c["dtype"] == "f32" else "bf16"
    y_ref, ht_ref = oracle_fwd(x)
    assert_parity(y, y_ref, kind, "y")
    assert_parity(ht, ht_ref, kind, "ht")
    ref = oracle.layer_core_bwd(npf(x["q"]), npf(x["k"]), npf(x["v"]), npf(x["conv_w"]), npf(x["alpha"]),
                                npf(x["z"]), npf(x["dout"]), norm_w=npf(x["norm_w"]),
                                **{k: npf(v) for k, v in gates(x).items()})
    keys = ["dxq", "dxk", "dxv", "dz", "dalpha", "dnorm_w"] + (["db", "dw"] if c["gpc"] else ["dbeta"])
    for key in keys:
        assert_parity(got[key], ref[key], kind, key)
    assert_parity(got["dconv_w"], ref["dconv_w"], kind, "dconv_w")


def test_norm_weights_of_one_rescale_the_ungated_output_rows_to_unit_rms():
    """With norm_w = 1, norm_eps = 0 and z large (swish(z) ~ z), y / z has rows of root mean square 1.
    (With eps > 0 a row's RMS is sqrt(m / (m + eps)), m its mean square: this layer's first outputs
    are small, as its conv weights have a standard deviation of 0.02.)"""
    B, T, Hk, Hv, d = 1, 64, 1, 2, 128
    x = inputs(B, T, Hk, Hv, d, False, False, "bf16", "f32", 102)
    x["norm_w"] = torch.ones(d, dtype=torch.bfloat16)
    x["z"] = torch.full_like(x["z"], 30.0)
    g = to_cuda(x)
    y, _, _ = gdn.gdn_layer_core_fwd(g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"], beta=g["beta"],
                                     norm_w=g["norm_w"], norm_eps=0.0, out_f32=True)
    torch.cuda.synchronize()
    rms = torch.sqrt(torch.mean((y / 30.0) ** 2, dim=-1))
    assert torch.allclose(rms, torch.ones_like(rms), atol=1e-4), rms.min().item()
