"""The seeded input recipe shared by the tests and the benchmark (inputs.py): shapes, dtypes,
ranges, determinism and the per-workload seeds.  CPU only, small sizes."""
import numpy as np
import torch

from gated_delta_rule_76_b200.inputs import (SEED_BASE, WORKLOADS, decode_initial_state, decode_inputs,
                                             decode_step_inputs, draw, workload_inputs)


def test_workloads_and_seeds():
    assert [w.index for w in WORKLOADS.values()] == [1, 2, 3, 4, 5]
    for w in WORKLOADS.values():
        assert w.seed == SEED_BASE + w.index
    gqa = WORKLOADS["gqa_layer_core_bf16"]
    assert (gqa.Hk, gqa.Hv, gqa.dk, gqa.dv) == (16, 128, 128, 128) and gqa.conv and gqa.swish_gate
    head = WORKLOADS["gdn2_fwd_bwd_bf16"]
    assert (head.B, head.T, head.Hk, head.dk) == (8, 4096, 16, 128) and head.tokens == 32768
    assert WORKLOADS["gdn2_decode_bf16"].tokens == 256 * 1024


def test_draw_shapes_dtypes_and_ranges():
    B, T, Hk, Hv, d = 2, 70, 1, 2, 16
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=True, gates_per_channel=True, dtype="bf16", seed=3,
             has_h0=True, swish_gate=True, with_dout=True, with_dht=True)
    assert x["q"].shape == (B, T, Hk, d) and x["v"].shape == (B, T, Hv, d)
    assert x["alpha"].shape == (B, T, Hv, d) and x["b"].shape == (B, T, Hv, d) and x["w"].shape == (B, T, Hv, d)
    assert x["z"].shape == x["dout"].shape == (B, T, Hv, d)
    assert x["h0"].shape == x["dht"].shape == (B, Hv, d, d)
    for key in ("q", "k", "v", "alpha", "b", "w", "z", "dout"):
        assert x[key].dtype == torch.bfloat16 and x[key].is_contiguous(), key
    assert x["h0"].dtype == torch.float32
    a = x["alpha"].double()
    # alpha = exp(-0.1 softplus(x)): in (0, 1), near 0.93 for x = 0
    assert float(a.min()) > 0.5 and float(a.max()) <= 1.0 and abs(float(a.median()) - np.exp(-0.1 * np.log(2))) < 0.02
    for key in ("b", "w"):
        v = x[key].double()
        assert float(v.min()) >= 0.0 and float(v.max()) <= 1.0 and abs(float(v.mean()) - 0.5) < 0.05
    # q, k rows of unit L2 norm (to the bf16 rounding of each entry)
    for key in ("q", "k"):
        n = x[key].double().norm(dim=-1)
        assert torch.allclose(n, torch.ones_like(n), atol=1e-2)
    assert abs(float(x["h0"].std()) - 0.1) < 0.01


def test_scalar_gates_conv_and_overrides():
    x = draw(1, 40, 2, 4, 8, 8, alpha_per_channel=False, gates_per_channel=False, dtype="bf16",
             gate_dtype="f32", seed=5, has_h0=False, conv=True, swish_gate=True, erase_scale=2.0, decay_scale=3.0)
    assert x["alpha"].shape == (1, 40, 4) and x["beta"].shape == (1, 40, 4) and "b" not in x and "h0" not in x
    assert x["alpha"].dtype == x["beta"].dtype == torch.float32
    assert float(x["beta"].max()) > 1.0 and float(x["beta"].max()) <= 2.0  # erase gates in [0, 2]
    assert float(x["alpha"].median()) < 0.3  # fast-forgetting decays
    assert x["conv_w"].shape == (2 * 2 * 8 + 4 * 8, 4) and abs(float(x["conv_w"].float().std()) - 0.02) < 0.005
    # the convolution's workloads leave q, k unnormalised (the layer normalises after the conv)
    n = x["q"].double().norm(dim=-1)
    assert float((n - 1.0).abs().max()) > 0.1


def test_draws_are_deterministic_and_seeded():
    kw = dict(alpha_per_channel=True, gates_per_channel=True, dtype="f32", has_h0=True)
    a = draw(1, 20, 1, 1, 8, 8, seed=7, **kw)
    b = draw(1, 20, 1, 1, 8, 8, seed=7, **kw)
    c = draw(1, 20, 1, 1, 8, 8, seed=8, **kw)
    for key in a:
        assert torch.equal(a[key], b[key]), key
    assert not torch.equal(a["q"], c["q"])
    # a named workload at reduced sizes draws with the workload's own seed and recipe
    w = workload_inputs("gdn2_fwd_bwd_bf16", B=1, T=16, Hk=1, Hv=1)
    ref = draw(1, 16, 1, 1, 128, 128, alpha_per_channel=True, gates_per_channel=True, dtype="bf16",
               gate_dtype="bf16", seed=SEED_BASE + 3, has_h0=True, with_dout=True)
    for key in ref:
        assert torch.equal(w[key], ref[key]), key


def test_decode_steps_draw_from_their_own_streams():
    one = decode_step_inputs("gdn2_decode_bf16", 5, B=3, Hk=1, Hv=2, dk=8, dv=8)
    stacked = decode_inputs("gdn2_decode_bf16", 7, threads=2, B=3, Hk=1, Hv=2, dk=8, dv=8)
    assert stacked["q"].shape == (7, 3, 1, 8) and stacked["alpha"].shape == (7, 3, 2, 8)
    for key in one:
        assert torch.equal(stacked[key][5], one[key]), key
    assert not torch.equal(stacked["q"][4], stacked["q"][5])
    s0 = decode_initial_state(B=3, Hv=2, dk=8, dv=8)
    assert s0.shape == (3, 2, 8, 8) and s0.dtype == torch.float32
