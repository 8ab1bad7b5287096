"""Gradients returned in the inputs' dtypes (grads_in_dtype): dq, dk, dv in bf16, the gates'
gradients in the gates' dtype, dh0 in fp32.  The kernels accumulate in fp32 and round once at the
store, so each bf16 gradient must be exactly the round-to-nearest-even of the fp32 gradient the
same call returns without the option; the fp32 gradients are checked against the oracle.  (A bf16
store alone costs up to 2^-8 of the largest entry, so the parity bound is taken on the fp32
values.)  Cases: channel gates with one key head per value head (dq, dk written directly) and with
two value heads per key head (fp32 partials summed, then rounded), scalar gates in fp32 and in
bf16, a fast-forgetting pair (the exact sequential kernel), the forward's cache, and gates given as
logits (their chain rule applied in place on the bf16 values: within two roundings).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_76_b200 import gdn
from gated_delta_rule_76_b200.inputs import draw
from oracle import oracle
from parity import assert_bf16_is_rounding, assert_parity, to_cuda

pytestmark = pytest.mark.gpu

KEYS_CH = ("dq", "dk", "dv", "dalpha", "db", "dw")
KEYS_SC = ("dq", "dk", "dv", "dalpha", "dbeta")


def gates(x):
    return dict(beta=x["beta"]) if "beta" in x else dict(b=x["b"], w=x["w"])


CASES = [
    dict(Hk=2, Hv=2, apc=True, gpc=True, gdt="bf16", fast=False, cache=False),
    dict(Hk=1, Hv=2, apc=True, gpc=True, gdt="bf16", fast=False, cache=False),
    dict(Hk=2, Hv=2, apc=True, gpc=True, gdt="bf16", fast=False, cache=True),
    dict(Hk=1, Hv=2, apc=False, gpc=False, gdt="f32", fast=False, cache=False),
    dict(Hk=2, Hv=2, apc=False, gpc=False, gdt="bf16", fast=False, cache=False),
    dict(Hk=2, Hv=2, apc=True, gpc=True, gdt="bf16", fast=True, cache=False),
]


def case_id(c):
    return (f"hk{c['Hk']}hv{c['Hv']}-{'ch' if c['apc'] else 'sc'}-{c['gdt']}"
            f"{'-fast' if c['fast'] else ''}{'-cache' if c['cache'] else ''}")


@pytest.mark.parametrize("c", CASES, ids=case_id)
def test_bf16_gradients_are_the_rounded_fp32_gradients(c):
    B, T, d = 2, 150, 128
    kw = dict(alpha_per_channel=c["apc"], gates_per_channel=c["gpc"], dtype="bf16", gate_dtype=c["gdt"],
              seed=131, has_h0=True, with_dout=True, with_dht=True)
    x = draw(B, T, c["Hk"], c["Hv"], d, d, **kw)
    if c["fast"]:
        x["alpha"][:, :, 1] = draw(B, T, c["Hk"], c["Hv"], d, d, decay_scale=3.0, **kw)["alpha"][:, :, 1]
    g = to_cuda(x)
    args = (g["q"], g["k"], g["v"], g["alpha"])
    common = dict(h0=g["h0"], grad_o=g["dout"], grad_ht=g["dht"], **gates(g))
    cache = None
    if c["cache"]:
        cache = torch.empty(gdn.gdn_chunk_fwd_cache_size(*args, h0=g["h0"], **gates(g)), dtype=torch.uint8,
                            device="cuda")
        gdn.gdn_chunk_fwd(*args, h0=g["h0"], bwd_cache=cache, **gates(g))
    g32 = gdn.gdn_chunk_bwd(*args, fwd_cache=cache, **common)
    g16 = gdn.gdn_chunk_bwd(*args, fwd_cache=cache, grads_in_dtype=True, **common)
    torch.cuda.synchronize()
    keys = KEYS_CH if c["gpc"] else KEYS_SC
    gate_dt = torch.bfloat16 if c["gdt"] == "bf16" else torch.float32
    for key in keys:
        want = torch.bfloat16 if key in ("dq", "dk", "dv") else gate_dt
        assert g16[key].dtype == want, (key, g16[key].dtype)
        if want == torch.bfloat16:
            assert_bf16_is_rounding(g16[key], g32[key], key)
        else:
            assert torch.equal(g16[key], g32[key]), key
    assert g16["dh0"].dtype == torch.float32 and torch.equal(g16["dh0"], g32["dh0"])
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], dout=x["dout"], dht=x["dht"], **gates(x))
    for key in keys + ("dh0",):
        assert_parity(g32[key], ref[key], "bf16", key)


def test_bf16_gradients_of_gate_logits():
    """Gates as logits: the chain rule runs in place on the rounded gate gradients, so each logit
    gradient is within two bf16 roundings of the fp32 call's; dalpha_scale (fp32) is summed from
    the rounded values and stays within the parity bound."""
    B, T, Hk, Hv, d = 2, 150, 1, 2, 128
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=True, gates_per_channel=True, dtype="bf16", gate_dtype="bf16",
             seed=133, has_h0=True, with_dout=True)
    gen = torch.Generator().manual_seed(134)
    for key in ("alpha", "b", "w"):
        x[key] = torch.randn(x[key].shape, generator=gen).to(torch.bfloat16)
    x["alpha_scale"] = (0.05 + 0.25 * torch.rand(Hv, generator=gen)).float()
    g = to_cuda(x)
    args = (g["q"], g["k"], g["v"], g["alpha"])
    common = dict(h0=g["h0"], grad_o=g["dout"], b=g["b"], w=g["w"], alpha_scale=g["alpha_scale"])
    g32 = gdn.gdn_chunk_bwd(*args, **common)
    g16 = gdn.gdn_chunk_bwd(*args, grads_in_dtype=True, **common)
    torch.cuda.synchronize()
    for key in ("dq", "dk", "dv"):
        assert_bf16_is_rounding(g16[key], g32[key], key)
    for key in ("dalpha", "db", "dw"):
        assert g16[key].dtype == torch.bfloat16
        a, b = g16[key].float(), g32[key]
        assert torch.all((a - b).abs() <= 2.0 ** -7 * b.abs() + 1e-30), key
    assert_parity(g16["dalpha_scale"], g32["dalpha_scale"].double().cpu().numpy(), "bf16", "dalpha_scale")


def test_bf16_gradients_unsupported_on_the_cuda_core_path():
    """bf16 inputs with dk = 64 take the CUDA-core backward, which returns fp32 gradients only."""
    x = draw(1, 64, 1, 1, 64, 64, alpha_per_channel=True, gates_per_channel=True, dtype="bf16", gate_dtype="bf16",
             seed=135, has_h0=False, with_dout=True)
    g = to_cuda(x)
    with pytest.raises(gdn.GdnError, match="grads_in_dtype"):
        gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"], grad_o=g["dout"],
                          grads_in_dtype=True)
    out = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"], grad_o=g["dout"])
    torch.cuda.synchronize()
    assert out["dq"].dtype == torch.float32 and np.isfinite(out["dq"].cpu().numpy()).all()
