"""GPU parity at the workloads' full sizes, in the launch configuration the benchmark times.

The GPU computes every (sequence, head) of the workload; the fp64 oracle recomputes a seeded
sample of at least 16 (sequence, head) pairs (each pair is an independent problem), and the
outputs, final states and gradients of those pairs are compared at the stated tolerances:
  * GDN-2 training step, B=8 T=4096 H=16 d=128 (bf16 inputs, fp32 state), as the benchmark runs
    it: the forward keeping the backward cache, then the backward reading it;
  * Gated DeltaNet forward with scalar gates, B=8 T=4096 H=16 d=128;
  * GQA layer core, B=2 T=16384, 16 key / 128 value heads (conv + SiLU + L2 + swish gate), and its
    training step (forward keeping the cache, backward) for one key head and its 8 value heads;
  * GDN-2 decode, 256 sequences x 1024 steps, H=16 d=128 (every step's output of the sampled
    sequences, and their final states).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_76_b200 import gdn
from gated_delta_rule_76_b200.inputs import (WORKLOADS, decode_initial_state, decode_inputs,
                                             workload_inputs)
from oracle import oracle
from parity import assert_bf16_is_rounding, assert_parity, npf

pytestmark = pytest.mark.gpu


def sample_pairs(B, H, n, seed):
    rng = np.random.default_rng(seed)
    flat = rng.choice(B * H, size=n, replace=False)
    return sorted((int(f) // H, int(f) % H) for f in flat)


def sample_heads_per_sequence(B, H, per_seq, seed):
    """{sequence: sorted heads}: `per_seq` distinct heads of every sequence, seeded."""
    rng = np.random.default_rng(seed)
    return {b: sorted(int(h) for h in rng.choice(H, size=per_seq, replace=False)) for b in range(B)}


def gate_kw(x, sl=slice(None)):
    if "beta" in x:
        return dict(beta=x["beta"][sl])
    return dict(b=x["b"][sl], w=x["w"][sl])


def test_gdn2_training_step_full_size():
    """The benchmark's step: gdn_chunk_fwd keeping the backward cache, then gdn_chunk_bwd reading
    it with the gradients in bf16; 2 heads of each of the 8 sequences (16 pairs) against the
    oracle's forward and reverse mode.  The output is also taken unrounded (fp32) from a forward
    without cache, and the gradients in fp32 from the same cache: the bf16 output and gradients must
    be their roundings, and the fp32 values meet the parity bound."""
    name = "gdn2_fwd_bwd_bf16"
    wl = WORKLOADS[name]
    x = workload_inputs(name, with_dout=True)
    g = {k: v.cuda() for k, v in x.items()}
    cache = torch.empty(gdn.gdn_chunk_fwd_cache_size(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], **gate_kw(g)),
                        dtype=torch.uint8, device="cuda")
    o16, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], bwd_cache=cache, **gate_kw(g))
    g16 = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], grad_o=g["dout"], fwd_cache=cache,
                            grads_in_dtype=True, **gate_kw(g))
    grads = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], grad_o=g["dout"], fwd_cache=cache,
                              **gate_kw(g))
    torch.cuda.synchronize()
    del cache
    for key in ("dq", "dk", "dv", "dalpha", "db", "dw"):
        assert_bf16_is_rounding(g16[key], grads[key], key)
    assert torch.equal(g16["dh0"], grads["dh0"])
    del g16
    o, ht32 = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], out_f32=True, **gate_kw(g))
    torch.cuda.synchronize()
    assert_bf16_is_rounding(o16, o, "o")
    assert torch.equal(ht, ht32)
    for b, heads in sample_heads_per_sequence(wl.B, wl.Hv, 2, seed=3).items():
        sl = slice(b, b + 1)
        xs = {k: v[sl] for k, v in x.items()}
        o_ref, ht_ref = oracle.fwd(xs["q"], xs["k"], xs["v"], xs["alpha"], h0=xs["h0"], pairs=heads,
                                   **gate_kw(xs))
        ref = oracle.bwd(xs["q"], xs["k"], xs["v"], xs["alpha"], h0=xs["h0"], dout=xs["dout"], pairs=heads,
                         **gate_kw(xs))
        for h in heads:
            assert_parity(o[b, :, h], o_ref[0, :, h], "bf16", f"o ({b},{h})")
            assert_parity(ht[b, h], ht_ref[0, h], "bf16", f"ht ({b},{h})")
            # identity head map: per-value-head q/k gradients are the q/k gradients of that head
            assert_parity(grads["dq"][b, :, h], ref["dq_v"][0, :, h], "bf16", f"dq ({b},{h})")
            assert_parity(grads["dk"][b, :, h], ref["dk_v"][0, :, h], "bf16", f"dk ({b},{h})")
            for key in ("dv", "dalpha", "db", "dw"):
                assert_parity(grads[key][b, :, h], ref[key][0, :, h], "bf16", f"{key} ({b},{h})")
            assert_parity(grads["dh0"][b, h], ref["dh0"][0, h], "bf16", f"dh0 ({b},{h})")


def test_gated_deltanet_scalar_forward_full_size():
    name = "gdn_fwd_scalar_bf16"
    wl = WORKLOADS[name]
    x = workload_inputs(name)
    g = {k: v.cuda() for k, v in x.items()}
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], beta=g["beta"], out_f32=True)
    torch.cuda.synchronize()
    for b, heads in sample_heads_per_sequence(wl.B, wl.Hv, 2, seed=4).items():
        sl = slice(b, b + 1)
        o_ref, ht_ref = oracle.fwd(x["q"][sl], x["k"][sl], x["v"][sl], x["alpha"][sl],
                                   beta=x["beta"][sl], pairs=heads)
        for h in heads:
            assert_parity(o[b, :, h], o_ref[0, :, h], "bf16", f"o ({b},{h})")
            assert_parity(ht[b, h], ht_ref[0, h], "bf16", f"ht ({b},{h})")


def test_gqa_layer_core_full_size():
    name = "gqa_layer_core_bf16"
    wl = WORKLOADS[name]
    x = workload_inputs(name)
    g = {k: v.cuda() for k, v in x.items()}
    y, ht, _ = gdn.gdn_layer_core_fwd(g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"],
                                      beta=g["beta"], out_f32=True)
    torch.cuda.synchronize()
    d, Hk, Hv = wl.dk, wl.Hk, wl.Hv
    w = npf(x["conv_w"])
    group = Hv // Hk
    for b, hvs in sample_heads_per_sequence(wl.B, wl.Hv, 8, seed=5).items():
        # the sampled value heads of sequence b with the key heads they read, as one oracle call
        hks = sorted({hv // group for hv in hvs})
        sl = slice(b, b + 1)
        cols = lambda base, heads: np.concatenate([np.arange(base + h * d, base + (h + 1) * d) for h in heads])
        q, _ = oracle.conv_silu(npf(x["q"][sl][:, :, hks]).reshape(1, -1, len(hks) * d), w[cols(0, hks)])
        k, _ = oracle.conv_silu(npf(x["k"][sl][:, :, hks]).reshape(1, -1, len(hks) * d), w[cols(Hk * d, hks)])
        v, _ = oracle.conv_silu(npf(x["v"][sl][:, :, hvs]).reshape(1, -1, len(hvs) * d), w[cols(2 * Hk * d, hvs)])
        q = oracle.l2norm(q.reshape(1, -1, len(hks), d))
        k = oracle.l2norm(k.reshape(1, -1, len(hks), d))
        o_ref, ht_ref = oracle.fwd(q, k, v.reshape(1, -1, len(hvs), d), npf(x["alpha"][sl][:, :, hvs]),
                                   beta=npf(x["beta"][sl][:, :, hvs]),
                                   head_map=[hks.index(hv // group) for hv in hvs])
        for i, hv in enumerate(hvs):
            y_ref = oracle.swish_gate(o_ref[0, :, i], npf(x["z"][b, :, hv]))
            assert_parity(y[b, :, hv], y_ref, "bf16", f"y ({b},{hv})")
            assert_parity(ht[b, hv], ht_ref[0, i], "bf16", f"ht ({b},{hv})")


def test_gqa_layer_training_step_full_size():
    """The layer's training step as the benchmark times it (forward keeping its cache, backward
    reading it) on the full workload.  The conv is depthwise and the key heads are independent, so
    the oracle recomputes one key head with its 8 value heads over both sequences exactly: every
    gradient of those channels, heads and conv weights is compared."""
    name = "gqa_layer_core_bf16"
    wl = WORKLOADS[name]
    x = workload_inputs(name, with_dout=True)
    g = {k: v.cuda() for k, v in x.items()}
    lin = (g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"])
    cache = torch.empty(gdn.gdn_layer_core_fwd_cache_size(*lin, beta=g["beta"]), dtype=torch.uint8, device="cuda")
    gdn.gdn_layer_core_fwd(*lin, beta=g["beta"], bwd_cache=cache, want_ht=False)
    got = gdn.gdn_layer_core_bwd(*lin, g["dout"], beta=g["beta"], fwd_cache=cache)
    torch.cuda.synchronize()
    del cache
    d, Hk, Hv = wl.dk, wl.Hk, wl.Hv
    group = Hv // Hk
    hk = int(np.random.default_rng(7).integers(Hk))
    hv = slice(hk * group, (hk + 1) * group)
    w = npf(x["conv_w"])
    rows = np.r_[hk * d:(hk + 1) * d, Hk * d + hk * d:Hk * d + (hk + 1) * d,
                 2 * Hk * d + hv.start * d:2 * Hk * d + hv.stop * d]
    ref = oracle.layer_core_bwd(npf(x["q"][:, :, hk:hk + 1]), npf(x["k"][:, :, hk:hk + 1]), npf(x["v"][:, :, hv]),
                                w[rows], npf(x["alpha"][:, :, hv]), npf(x["z"][:, :, hv]), npf(x["dout"][:, :, hv]),
                                beta=npf(x["beta"][:, :, hv]))
    assert_parity(got["dxq"][:, :, hk:hk + 1], ref["dxq"], "bf16", f"dxq (key head {hk})")
    assert_parity(got["dxk"][:, :, hk:hk + 1], ref["dxk"], "bf16", f"dxk (key head {hk})")
    for key in ("dxv", "dz", "dalpha", "dbeta"):
        assert_parity(got[key][:, :, hv], ref[key], "bf16", key)
    assert_parity(got["dh0"][:, hv], ref["dh0"], "bf16", "dh0")
    assert_parity(got["dconv_w"].cpu()[torch.as_tensor(rows)], ref["dconv_w"], "bf16", "dconv_w")


def test_gdn2_decode_1024_steps_full_size():
    name = "gdn2_decode_bf16"
    wl = WORKLOADS[name]
    steps = wl.decode_steps
    xs = decode_inputs(name, steps)
    s0 = decode_initial_state(name)
    g = {k: v.cuda() for k, v in xs.items()}
    state = s0.cuda()
    o = torch.empty((steps, wl.B, wl.Hv, wl.dv), dtype=torch.float32, device="cuda")
    for s in range(steps):
        gdn.gdn_decode_step(state, g["q"][s], g["k"][s], g["v"][s], g["alpha"][s], b=g["b"][s], w=g["w"][s],
                            o=o[s])
    torch.cuda.synchronize()
    for n, h in sample_pairs(wl.B, wl.Hv, 16, seed=6):
        # The sampled sequence's 1024 steps as one sequence (T decode steps == one forward).
        seq = {k: v[:, n:n + 1].transpose(0, 1).contiguous() for k, v in xs.items()}
        o_ref, st_ref = oracle.fwd(seq["q"], seq["k"], seq["v"], seq["alpha"], b=seq["b"], w=seq["w"],
                                   h0=s0[n:n + 1], pairs=[h])
        assert_parity(o[:, n, h], o_ref[0, :, h], "bf16", f"o ({n},{h})")
        assert_parity(state[n, h], st_ref[0, h], "bf16", f"state ({n},{h})")
