"""GPU parity of the single-token decode step (with and without the fused short convolution
and swish gate) and of the GQA layer core, against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from gated_delta_rule_76_b200 import gdn
from gated_delta_rule_76_b200.inputs import draw
from oracle import oracle
from parity import assert_bf16_is_rounding, assert_parity, npf, to_cuda

pytestmark = pytest.mark.gpu


def step_inputs(rng_seed, N, Hk, Hv, d, apc, gpc, dtype, gate_dtype, steps):
    x = draw(N, steps, Hk, Hv, d, d, alpha_per_channel=apc, gates_per_channel=gpc, dtype=dtype,
             gate_dtype=gate_dtype, seed=rng_seed, has_h0=True)
    return x


@pytest.mark.parametrize("N,Hk,Hv,d,apc,gpc,dtype,gdt", [
    (5, 2, 4, 128, True, True, "bf16", "bf16"),
    (3, 1, 2, 64, True, True, "f32", "f32"),
    (4, 2, 2, 128, False, False, "bf16", "f32"),
    (2, 2, 4, 64, True, False, "bf16", "bf16"),
])
def test_decode_steps_match_oracle(N, Hk, Hv, d, apc, gpc, dtype, gdt):
    steps = 6
    x = step_inputs(11, N, Hk, Hv, d, apc, gpc, dtype, gdt, steps)
    g = to_cuda(x)
    state = g["h0"].clone()
    ref_state = npf(x["h0"])
    kind = "f32" if dtype == "f32" else "bf16"
    for t in range(steps):
        tk = lambda src, key: src[key][:, t].contiguous()
        gk = dict(beta=tk(g, "beta")) if not gpc else dict(b=tk(g, "b"), w=tk(g, "w"))
        xk = dict(beta=tk(x, "beta")) if not gpc else dict(b=tk(x, "b"), w=tk(x, "w"))
        s16 = state.clone()
        o = gdn.gdn_decode_step(state, tk(g, "q"), tk(g, "k"), tk(g, "v"), tk(g, "alpha"), scale=0.9,
                                out_f32=True, **gk)
        o_ref, ref_state = oracle.decode_step(ref_state, tk(x, "q"), tk(x, "k"), tk(x, "v"),
                                              tk(x, "alpha"), scale=0.9, **xk)
        assert_parity(o, o_ref, kind, f"o step {t}")
        if kind == "bf16":
            o16 = gdn.gdn_decode_step(s16, tk(g, "q"), tk(g, "k"), tk(g, "v"), tk(g, "alpha"),
                                      scale=0.9, **gk)
            assert_bf16_is_rounding(o16, o, f"o step {t}")
            assert torch.equal(s16, state)
    assert_parity(state, ref_state, kind, "state")


@pytest.mark.parametrize("N,Hk,Hv,d,steps", [
    (3, 2, 4, 64, 5),
    (8, 2, 16, 128, 8),  # the layer's head width and an 8-value-head group per key head
])
def test_decode_with_conv_and_swish_gate(N, Hk, Hv, d, steps):
    cch = 2 * Hk * d + Hv * d
    x = draw(N, steps, Hk, Hv, d, d, alpha_per_channel=True, gates_per_channel=True, dtype="bf16",
             gate_dtype="bf16", seed=21, has_h0=True, conv=True, swish_gate=True)
    g = to_cuda(x)
    gen = torch.Generator().manual_seed(4)
    hist0 = torch.randn((N, cch, 3), generator=gen).to(torch.bfloat16)
    conv_state = hist0.cuda().clone()
    state = g["h0"].clone()
    ref_state, ref_hist = npf(x["h0"]), npf(hist0)
    w = npf(x["conv_w"])
    for t in range(steps):
        tk = lambda src, key: src[key][:, t].contiguous()
        o = gdn.gdn_decode_step(state, tk(g, "q"), tk(g, "k"), tk(g, "v"), tk(g, "alpha"),
                                b=tk(g, "b"), w=tk(g, "w"), conv_state=conv_state,
                                conv_w=g["conv_w"], z=tk(g, "z"), out_f32=True)
        # Oracle: conv (kernel 4) + SiLU over [history, new input], L2 on q, k, then the step.
        raw = np.concatenate([npf(tk(x, "q")).reshape(N, -1), npf(tk(x, "k")).reshape(N, -1),
                              npf(tk(x, "v")).reshape(N, -1)], axis=1)[:, None, :]
        y, ref_hist = oracle.conv_silu(raw, w, hist=ref_hist)
        y = y[:, 0]
        qc = oracle.l2norm(y[:, :Hk * d].reshape(N, Hk, d))
        kc = oracle.l2norm(y[:, Hk * d:2 * Hk * d].reshape(N, Hk, d))
        vc = y[:, 2 * Hk * d:].reshape(N, Hv, d)
        o_ref, ref_state = oracle.decode_step(ref_state, qc, kc, vc, tk(x, "alpha"), b=tk(x, "b"),
                                              w=tk(x, "w"))
        assert_parity(o, oracle.swish_gate(o_ref, tk(x, "z")), "bf16", f"y step {t}")
        assert np.array_equal(npf(conv_state), ref_hist), "conv state"
    assert_parity(state, ref_state, "bf16", "state")


@pytest.mark.parametrize("apc,gpc", [(False, False), (True, True)])
def test_layer_core_matches_oracle(apc, gpc):
    B, T, Hk, Hv, d = 2, 150, 2, 4, 64
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=apc, gates_per_channel=gpc, dtype="bf16",
             gate_dtype="f32", seed=31, has_h0=False, conv=True, swish_gate=True)
    g = to_cuda(x)
    gk = dict(beta=g["beta"]) if not gpc else dict(b=g["b"], w=g["w"])
    y, ht, cs = gdn.gdn_layer_core_fwd(g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"],
                                       want_conv_state=True, out_f32=True, **gk)
    y16, _, _ = gdn.gdn_layer_core_fwd(g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"], **gk)
    torch.cuda.synchronize()
    assert_bf16_is_rounding(y16, y, "y")
    xk = dict(beta=x["beta"]) if not gpc else dict(b=x["b"], w=x["w"])
    if gpc:
        # layer_core_fwd of the oracle takes scalar beta; compose by hand for channel gates
        cq = Hk * d
        w = npf(x["conv_w"])
        q, _ = oracle.conv_silu(npf(x["q"]).reshape(B, T, cq), w[:cq])
        k, _ = oracle.conv_silu(npf(x["k"]).reshape(B, T, cq), w[cq:2 * cq])
        v, _ = oracle.conv_silu(npf(x["v"]).reshape(B, T, Hv * d), w[2 * cq:])
        o_ref, ht_ref = oracle.fwd(oracle.l2norm(q.reshape(B, T, Hk, d)),
                                   oracle.l2norm(k.reshape(B, T, Hk, d)), v.reshape(B, T, Hv, d),
                                   x["alpha"], **xk)
        y_ref = oracle.swish_gate(o_ref, x["z"])
    else:
        y_ref, ht_ref = oracle.layer_core_fwd(x["q"], x["k"], x["v"], x["conv_w"], x["alpha"],
                                              x["beta"], x["z"])
    assert_parity(y, y_ref, "bf16", "y")
    assert_parity(ht, ht_ref, "bf16", "ht")
    raw = torch.cat([x["q"].reshape(B, T, -1), x["k"].reshape(B, T, -1), x["v"].reshape(B, T, -1)], 2)
    assert torch.equal(cs.cpu(), raw[:, -3:].permute(0, 2, 1).contiguous())


@pytest.mark.parametrize("B,T,Hk,Hv,gdt", [(1, 200, 2, 8, "f32"), (2, 129, 1, 2, "bf16"), (1, 64, 1, 1, "f32")])
def test_layer_core_tensor_core_path(B, T, Hk, Hv, gdt):
    """d = 128 with scalar gates: the conv kernel hands the tensor-core forward its fp32 outputs as
    bf16 hi/lo pairs (three launches: conv, chunk forward, and the sequential kernel for pairs
    outside the decay range, which returns at once here).  Several chunks, a ragged tail, GQA."""
    d = 128
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=False, gates_per_channel=False, dtype="bf16",
             gate_dtype=gdt, seed=37, has_h0=True, conv=True, swish_gate=True)
    g = to_cuda(x)
    n0 = gdn.kernel_launches()
    y, ht, _ = gdn.gdn_layer_core_fwd(g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"], beta=g["beta"],
                                      h0=g["h0"], scale=0.8, out_f32=True)
    torch.cuda.synchronize()
    assert gdn.kernel_launches() - n0 == 3, "conv + tensor-core forward + range fallback"
    y16, _, _ = gdn.gdn_layer_core_fwd(g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"], beta=g["beta"],
                                       h0=g["h0"], scale=0.8)
    torch.cuda.synchronize()
    assert_bf16_is_rounding(y16, y, "y")
    y_ref, ht_ref = oracle.layer_core_fwd(x["q"], x["k"], x["v"], x["conv_w"], x["alpha"], x["beta"], x["z"],
                                          scale=0.8, h0=x["h0"])
    assert_parity(y, y_ref, "bf16", "y")
    assert_parity(ht, ht_ref, "bf16", "ht")


def test_decode_negative_eigenvalue_gates():
    """Erase gates in [0, 2] (the explainer's note under «Réunir les deux») through the decode
    step, each side carrying its own state."""
    N, Hk, Hv, d, steps = 3, 1, 2, 128, 6
    x = draw(N, steps, Hk, Hv, d, d, alpha_per_channel=True, gates_per_channel=True, dtype="bf16",
             gate_dtype="bf16", seed=43, has_h0=True, erase_scale=2.0)
    assert float(x["b"].float().max()) > 1.5
    g = to_cuda(x)
    state = g["h0"].clone()
    ref_state = npf(x["h0"])
    for t in range(steps):
        tk = lambda src, key: src[key][:, t].contiguous()
        o = gdn.gdn_decode_step(state, tk(g, "q"), tk(g, "k"), tk(g, "v"), tk(g, "alpha"), b=tk(g, "b"),
                                w=tk(g, "w"), out_f32=True)
        o_ref, ref_state = oracle.decode_step(ref_state, tk(x, "q"), tk(x, "k"), tk(x, "v"), tk(x, "alpha"),
                                              b=tk(x, "b"), w=tk(x, "w"))
        assert_parity(o, o_ref, "bf16", f"o step {t}")
    assert_parity(state, ref_state, "bf16", "state")


@pytest.mark.parametrize("B,T,Hk,Hv,d,gpc,gdt,dt,h0", [
    (2, 150, 2, 4, 64, False, "f32", "bf16", True),    # GQA, scalar gates, ragged tail
    (1, 130, 1, 2, 128, False, "bf16", "bf16", True),  # d = 128 with h0: CUDA-core recurrence backward
    (2, 200, 2, 4, 128, False, "f32", "bf16", True),   # same, GQA, fp32 gates, ragged tail
    (1, 130, 1, 2, 128, False, "bf16", "bf16", False),  # d = 128 without h0: tensor-core backward (hi/lo)
    (2, 200, 2, 4, 128, False, "f32", "bf16", False),   # same, GQA, fp32 gates, ragged tail, dht given
    (1, 100, 1, 2, 64, True, "bf16", "bf16", True),    # channel gates
    (1, 70, 1, 1, 64, False, "f32", "f32", True),      # fp32 tensors
])
def test_layer_core_backward_matches_oracle(B, T, Hk, Hv, d, gpc, gdt, dt, h0):
    """gdn_layer_core_bwd against the oracle's reverse mode of the layer (itself pinned by finite
    differences): gradients of the conv inputs, the conv weights, the gates, z and h0."""
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=gpc, gates_per_channel=gpc, dtype=dt,
             gate_dtype=gdt, seed=61, has_h0=h0, conv=True, swish_gate=True, with_dout=True, with_dht=True)
    g = to_cuda(x)
    gk = dict(beta=g["beta"]) if not gpc else dict(b=g["b"], w=g["w"])
    xk = dict(beta=x["beta"]) if not gpc else dict(b=x["b"], w=x["w"])
    got = gdn.gdn_layer_core_bwd(g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"], g["dout"],
                                 h0=g.get("h0"), grad_ht=g["dht"], scale=0.8, **gk)
    torch.cuda.synchronize()
    ref = oracle.layer_core_bwd(x["q"], x["k"], x["v"], x["conv_w"], x["alpha"], x["z"], x["dout"],
                                h0=x.get("h0"), dht=x["dht"], scale=0.8, **xk)
    kind = "f32" if dt == "f32" else "bf16"
    for key in ["dxq", "dxk", "dxv", "dconv_w", "dalpha", "dz", "dh0"] + (["db", "dw"] if gpc else ["dbeta"]):
        assert_parity(got[key], ref[key], kind, key)


@pytest.mark.parametrize("B,T,Hk,Hv,gdt", [(2, 200, 2, 4, "f32"), (1, 64, 1, 1, "bf16")])
def test_layer_core_backward_from_forward_cache(B, T, Hk, Hv, gdt):
    """A layer forward keeping its cache, then a backward reading it: y and every gradient are
    bit for bit those of the calls without a cache (the same kernels on the same values), and the
    gradients match the oracle."""
    x = draw(B, T, Hk, Hv, 128, 128, alpha_per_channel=False, gates_per_channel=False, dtype="bf16",
             gate_dtype=gdt, seed=67, has_h0=False, conv=True, swish_gate=True, with_dout=True, with_dht=True)
    g = to_cuda(x)
    args = (g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"])
    n = gdn.gdn_layer_core_fwd_cache_size(*args, beta=g["beta"], scale=0.8)
    assert n > 0
    cache = torch.empty(n, dtype=torch.uint8, device="cuda")
    y_c, ht_c, _ = gdn.gdn_layer_core_fwd(*args, beta=g["beta"], scale=0.8, out_f32=True, bwd_cache=cache)
    y, ht, _ = gdn.gdn_layer_core_fwd(*args, beta=g["beta"], scale=0.8, out_f32=True)
    got_c = gdn.gdn_layer_core_bwd(*args, g["dout"], beta=g["beta"], grad_ht=g["dht"], scale=0.8, fwd_cache=cache)
    got = gdn.gdn_layer_core_bwd(*args, g["dout"], beta=g["beta"], grad_ht=g["dht"], scale=0.8)
    torch.cuda.synchronize()
    assert torch.equal(y_c, y) and torch.equal(ht_c, ht)
    keys = ["dxq", "dxk", "dxv", "dconv_w", "dalpha", "dz", "dh0", "dbeta"]
    for key in keys:
        assert torch.equal(got_c[key], got[key]), key
    ref = oracle.layer_core_bwd(x["q"], x["k"], x["v"], x["conv_w"], x["alpha"], x["z"], x["dout"],
                                dht=x["dht"], scale=0.8, beta=x["beta"])
    for key in keys:
        assert_parity(got_c[key], ref[key], "bf16", key)
