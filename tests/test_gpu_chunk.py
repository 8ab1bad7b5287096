"""GPU parity of the chunkwise forward and backward against the fp64 oracle, through the C ABI,
on small seeded inputs that span several chunks and a ragged tail, plus edge cases."""
import numpy as np
import pytest
import torch

from gated_delta_rule_76_b200 import gdn
from gated_delta_rule_76_b200.inputs import draw, workload_inputs
from oracle import oracle
from parity import assert_bf16_is_rounding, assert_parity, kind_of, to_cuda

pytestmark = pytest.mark.gpu

CASES = {
    # name: (B, T, Hk, Hv, d, alpha per channel, gates per channel, dtype, gate dtype, h0, scale)
    "gdn2_bf16_ragged": (2, 200, 2, 2, 128, True, True, "bf16", "bf16", True, 1.0),
    "gdn_scalar_bf16_f32gates_gqa": (1, 130, 1, 4, 128, False, False, "bf16", "f32", True, 1.0),
    "kda_f32_d128": (1, 65, 2, 2, 128, True, False, "f32", "f32", True, 0.5),
    # tensor-core path, the two mixed gate forms (channel alpha + scalar beta; scalar alpha + b, w)
    "kda_bf16_d128": (1, 140, 2, 2, 128, True, False, "bf16", "bf16", True, 0.8),
    "gdn2_scalar_alpha_bf16_d128_gqa": (1, 100, 1, 2, 128, False, True, "bf16", "bf16", True, 1.0),
    "gdn2_scalar_alpha_bf16_d64": (3, 97, 2, 2, 64, False, True, "bf16", "bf16", False, 1.0),
    "gdn2_f32_d64_gqa": (2, 150, 1, 2, 64, True, True, "f32", "f32", True, 1.0),
    "one_token": (2, 1, 1, 1, 128, True, True, "bf16", "bf16", True, 1.0),
    "chunk_minus_one": (1, 63, 1, 1, 128, True, True, "bf16", "bf16", True, 1.0),
    "exact_chunk": (1, 64, 1, 1, 64, True, True, "f32", "f32", True, 1.0),
}


def make(name, with_dout=False, seed=7):
    B, T, Hk, Hv, d, apc, gpc, dt, gdt, h0, scale = CASES[name]
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=apc, gates_per_channel=gpc, dtype=dt,
             gate_dtype=gdt, seed=seed, has_h0=h0, with_dout=with_dout, with_dht=with_dout)
    return x, scale


def gate_kw(x):
    return dict(beta=x["beta"]) if "beta" in x else dict(b=x["b"], w=x["w"])


@pytest.mark.parametrize("name", list(CASES))
def test_chunk_fwd_matches_oracle(name):
    x, scale = make(name)
    g = to_cuda(x)
    kind = kind_of(x["q"])
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g.get("h0"), scale=scale,
                              out_f32=True, **gate_kw(g))
    torch.cuda.synchronize()
    o_ref, ht_ref = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], h0=x.get("h0"), scale=scale,
                               **gate_kw(x))
    assert_parity(o, o_ref, kind, "o")
    assert_parity(ht, ht_ref, kind, "ht")
    if kind == "bf16":
        o16, ht16 = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g.get("h0"),
                                      scale=scale, **gate_kw(g))
        assert_bf16_is_rounding(o16, o, "o")
        assert torch.equal(ht16, ht)


def test_tiny_fp32_workload_fwd():
    """The 1 x 256 x 2 x 64 fp32 GDN-2 workload at the fp32 tolerance."""
    x = workload_inputs("gdn2_fwd_tiny_f32")
    g = to_cuda(x)
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"])
    o_ref, ht_ref = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"])
    assert_parity(o, o_ref, "f32", "o")
    assert_parity(ht, ht_ref, "f32", "ht")


@pytest.mark.parametrize("name", list(CASES))
def test_chunk_bwd_matches_oracle(name):
    x, scale = make(name, with_dout=True)
    g = to_cuda(x)
    grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], h0=g.get("h0"), scale=scale,
                              grad_o=g["dout"], grad_ht=g["dht"], **gate_kw(g))
    torch.cuda.synchronize()
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], h0=x.get("h0"), scale=scale,
                     dout=x["dout"], dht=x["dht"], **gate_kw(x))
    kind = kind_of(x["q"])
    for key in ["dq", "dk", "dv", "dalpha", "dh0"] + (["dbeta"] if "beta" in x else ["db", "dw"]):
        assert_parity(grads[key], ref[key], kind, key)


def test_swish_gated_forward():
    x, _ = make("gdn2_bf16_ragged")
    z = torch.randn(x["v"].shape, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    g = to_cuda(x)
    y, _ = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"], h0=g["h0"],
                             z=z.cuda(), out_f32=True)
    o_ref, _ = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"])
    assert_parity(y, oracle.swish_gate(o_ref, z), "bf16", "y")
    y16, _ = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"], h0=g["h0"],
                               z=z.cuda())
    assert_bf16_is_rounding(y16, y, "y")


def test_explicit_head_map():
    B, T, Hk, Hv, d = 1, 90, 2, 4, 64
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=True, gates_per_channel=True, dtype="f32",
             gate_dtype="f32", seed=5, has_h0=True, with_dout=True)
    hmap = [1, 0, 0, 1]
    g = to_cuda(x)
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"], h0=g["h0"],
                              head_map=hmap)
    o_ref, ht_ref = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"],
                               head_map=hmap)
    assert_parity(o, o_ref, "f32", "o")
    grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"], h0=g["h0"],
                              head_map=hmap, grad_o=g["dout"])
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"],
                     head_map=hmap, dout=x["dout"])
    for key in ["dq", "dk", "dv", "dalpha", "db", "dw", "dh0"]:
        assert_parity(grads[key], ref[key], "f32", key)


def test_split_sequence_carry_on_gpu():
    """Two calls with the first call's final state as the second's h0 equal one call."""
    x, _ = make("gdn2_bf16_ragged")
    g = to_cuda(x)
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"], h0=g["h0"],
                              out_f32=True)
    cut = 77
    sl = lambda t, a, b_: t[:, a:b_].contiguous()
    o1, h1 = gdn.gdn_chunk_fwd(sl(g["q"], 0, cut), sl(g["k"], 0, cut), sl(g["v"], 0, cut),
                               sl(g["alpha"], 0, cut), b=sl(g["b"], 0, cut), w=sl(g["w"], 0, cut),
                               h0=g["h0"], out_f32=True)
    o2, h2 = gdn.gdn_chunk_fwd(sl(g["q"], cut, None), sl(g["k"], cut, None), sl(g["v"], cut, None),
                               sl(g["alpha"], cut, None), b=sl(g["b"], cut, None),
                               w=sl(g["w"], cut, None), h0=h1, out_f32=True)
    assert_parity(torch.cat([o1, o2], 1), o, "bf16", "o split")
    assert_parity(h2, ht, "bf16", "ht split")


def test_zero_length_sequence_copies_state():
    x, _ = make("one_token")
    g = to_cuda(x)
    e = lambda t: t[:, :0].contiguous()
    o, ht = gdn.gdn_chunk_fwd(e(g["q"]), e(g["k"]), e(g["v"]), e(g["alpha"]), b=e(g["b"]),
                              w=e(g["w"]), h0=g["h0"])
    assert o.numel() == 0
    assert torch.equal(ht, g["h0"])


def test_invalid_arguments_raise_on_gpu():
    x, _ = make("one_token")
    g = to_cuda(x)
    with pytest.raises(gdn.GdnError, match="INVALID_ARG"):
        gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"], h0=g["h0"],
                          o=g["v"])
    with pytest.raises(gdn.GdnError):
        gdn.gdn_chunk_fwd(g["q"].cpu(), g["k"], g["v"], g["alpha"], b=g["b"], w=g["w"])


@pytest.mark.parametrize("name", ["gdn2_bf16_ragged", "gdn_scalar_bf16_f32gates_gqa", "one_token",
                                  "chunk_minus_one"])
def test_bwd_from_forward_cache_matches_recompute(name):
    """A forward that fills the cache gives the same o, ht; a backward given the cache gives the
    same gradients as one that recomputes the forward (the same kernels on the same inputs)."""
    x, scale = make(name, with_dout=True)
    g = to_cuda(x)
    kw = dict(h0=g.get("h0"), scale=scale, **gate_kw(g))
    nbytes = gdn.gdn_chunk_fwd_cache_size(g["q"], g["k"], g["v"], g["alpha"], **kw)
    assert nbytes > 0
    cache = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], out_f32=True, bwd_cache=cache, **kw)
    o_ref, ht_ref = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], out_f32=True, **kw)
    assert torch.equal(o, o_ref) and torch.equal(ht, ht_ref)
    with_cache = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], grad_o=g["dout"], grad_ht=g["dht"],
                                   fwd_cache=cache, **kw)
    recompute = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], grad_o=g["dout"], grad_ht=g["dht"], **kw)
    torch.cuda.synchronize()
    for key in with_cache:
        assert torch.equal(with_cache[key], recompute[key]), key
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], h0=x.get("h0"), scale=scale, dout=x["dout"],
                     dht=x["dht"], **gate_kw(x))
    for key in ["dq", "dk", "dv", "dalpha", "dh0"] + (["dbeta"] if "beta" in x else ["db", "dw"]):
        assert_parity(with_cache[key], ref[key], "bf16", key)


def test_forward_cache_is_refused_off_the_tensor_core_path():
    x, scale = make("kda_f32_d128", with_dout=True)
    g = to_cuda(x)
    kw = dict(h0=g.get("h0"), scale=scale, **gate_kw(g))
    assert gdn.gdn_chunk_fwd_cache_size(g["q"], g["k"], g["v"], g["alpha"], **kw) == 0
    cache = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(gdn.GdnError, match="UNSUPPORTED"):
        gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], bwd_cache=cache, **kw)


@pytest.mark.parametrize("B,T,Hk,Hv,d,apc,gpc,dt", [
    (1, 150, 2, 2, 128, True, True, "bf16"),     # tensor-core path, channel gates
    (1, 130, 1, 2, 128, False, False, "bf16"),   # tensor-core path, scalar beta
    (1, 100, 1, 1, 64, True, True, "f32"),       # CUDA-core path
])
def test_negative_eigenvalue_gates(B, T, Hk, Hv, d, apc, gpc, dt):
    """Erase gates b, beta in [0, 2] (the explainer's note under «Réunir les deux»): forward and
    backward against the oracle, the kernels unchanged."""
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=apc, gates_per_channel=gpc, dtype=dt, gate_dtype=dt,
             seed=41, has_h0=True, with_dout=True, with_dht=True, erase_scale=2.0)
    gk = gate_kw(x)
    assert float((gk["b"] if gpc else gk["beta"]).float().max()) > 1.5
    g = to_cuda(x)
    kind = kind_of(x["q"])
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], out_f32=True, **gate_kw(g))
    o_ref, ht_ref = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], **gk)
    assert_parity(o, o_ref, kind, "o")
    assert_parity(ht, ht_ref, kind, "ht")
    grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], grad_o=g["dout"],
                              grad_ht=g["dht"], **gate_kw(g))
    torch.cuda.synchronize()
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], dout=x["dout"], dht=x["dht"], **gk)
    for key in ["dq", "dk", "dv", "dalpha", "dh0"] + (["db", "dw"] if gpc else ["dbeta"]):
        assert_parity(grads[key], ref[key], kind, key)
