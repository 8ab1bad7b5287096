"""Token strides (gdn_strides): inputs given as slices of one fused projection buffer, with their
tokens evenly spaced, must give bit for bit what the same call gives on dense copies of them.
The chunk and layer calls copy each strided input into their workspace before their kernels run,
so their results are the dense call's exactly; the decode step reads strided inputs in place,
element by element, so its results are the dense call's exactly as well.  The dense calls are
checked against the oracle by the other GPU tests; one case here checks the oracle too.  Cases
cover both forward paths (tensor cores: bf16, d = 128; CUDA cores: fp32 or d = 64), the
backward with and without the forward's cache, slices that start at an odd element (2-byte
copy units), the segment map, the no-alloc forward, the layer calls and the decode step."""
import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_76_b200 import gdn
from gated_delta_rule_76_b200.inputs import draw
from oracle import oracle
from parity import assert_bf16_is_rounding, assert_parity, to_cuda

pytestmark = pytest.mark.gpu


def fused(tensors, lead=2, pad=8, offset=0):
    """Views of the given token-major tensors as column slices of one buffer per dtype
    ([tokens, C] with `pad` spare elements after each slice and `offset` before the first), holding
    the same values.  `lead` is the number of token dimensions."""
    out, groups = {}, {}
    for name, t in tensors.items():
        if t is not None:
            groups.setdefault(t.dtype, []).append(name)
    for dt, names in groups.items():
        rows = int(np.prod(tensors[names[0]].shape[:lead]))
        widths = [int(np.prod(tensors[n].shape[lead:])) for n in names]
        C = offset + sum(w + pad for w in widths)
        buf = torch.full((rows, C), float("nan"), dtype=dt, device="cuda")
        col = offset
        for n, w in zip(names, widths):
            t = tensors[n]
            buf[:, col:col + w] = t.reshape(rows, w)
            out[n] = buf[:, col:col + w].view(t.shape)
            assert not out[n].is_contiguous() and torch.equal(out[n], t)
            col += w + pad
    return out


def gates(x):
    return dict(beta=x["beta"]) if "beta" in x else dict(b=x["b"], w=x["w"])


FWD_CASES = [
    dict(Hk=2, Hv=2, d=128, apc=True, gpc=True, dt="bf16", gdt="bf16", z=False, offset=0),   # tensor cores
    dict(Hk=1, Hv=2, d=128, apc=False, gpc=False, dt="bf16", gdt="f32", z=True, offset=1),   # odd start
    dict(Hk=2, Hv=4, d=64, apc=True, gpc=True, dt="bf16", gdt="bf16", z=False, offset=3),    # CUDA cores
    dict(Hk=1, Hv=1, d=64, apc=True, gpc=False, dt="f32", gdt="f32", z=True, offset=0),      # fp32
]


def case_id(c):
    return f"hk{c['Hk']}hv{c['Hv']}d{c['d']}-{c['dt']}-{c['gdt']}{'-z' if c['z'] else ''}-off{c['offset']}"


def inputs(c, B=2, T=150, seed=301):
    x = draw(B, T, c["Hk"], c["Hv"], c["d"], c["d"], alpha_per_channel=c["apc"], gates_per_channel=c["gpc"],
             dtype=c["dt"], gate_dtype=c["gdt"], seed=seed, has_h0=True, swish_gate=c["z"], with_dout=True,
             with_dht=True)
    return x, to_cuda(x)


def strided_inputs(g, c):
    names = ("q", "k", "v", "alpha", "b", "w", "beta", "z")
    return fused({n: g.get(n) for n in names if g.get(n) is not None}, offset=c["offset"])


@pytest.mark.parametrize("c", FWD_CASES, ids=case_id)
def test_forward_and_backward_on_strided_inputs(c):
    x, g = inputs(c)
    s = strided_inputs(g, c)
    z, zs = g.get("z"), s.get("z")
    o, ht = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], z=z, **gates(g))
    os_, hts = gdn.gdn_chunk_fwd(s["q"], s["k"], s["v"], s["alpha"], h0=g["h0"], z=zs, **gates(s))
    common = dict(h0=g["h0"], grad_o=g["dout"], grad_ht=g["dht"])
    gd = gdn.gdn_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], **common, **gates(g))
    gs = gdn.gdn_chunk_bwd(s["q"], s["k"], s["v"], s["alpha"], **common, **gates(s))
    torch.cuda.synchronize()
    assert torch.equal(o, os_) and torch.equal(ht, hts)
    for key, val in gd.items():
        assert torch.equal(val, gs[key]), key
    if c["offset"] == 1:
        # this case also against the oracle: the gated output unrounded (out_f32), whose bf16
        # rounding the strided call returned, and the final state
        y32, _ = gdn.gdn_chunk_fwd(s["q"], s["k"], s["v"], s["alpha"], h0=g["h0"], z=zs, out_f32=True, **gates(s))
        o_ref, ht_ref = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], **gates(x))
        assert_parity(y32, oracle.swish_gate(o_ref, x["z"]), "bf16", "o")
        assert_bf16_is_rounding(os_, y32, "o")
        assert_parity(hts, ht_ref, "bf16", "ht")


def test_workspace_grows_by_the_dense_copies():
    c = FWD_CASES[0]
    x, g = inputs(c, B=1, T=64)
    s = strided_inputs(g, c)
    lib = gdn.load()
    a_dense, keep1 = gdn.fwd_args(g["q"], g["k"], g["v"], g["alpha"], **gates(g))
    a_strided, keep2 = gdn.fwd_args(s["q"], s["k"], s["v"], s["alpha"], **gates(s))
    dense = lib.gdn_chunk_fwd_workspace_size(ctypes.byref(a_dense))
    strided = lib.gdn_chunk_fwd_workspace_size(ctypes.byref(a_strided))
    copies = sum(-(-t.numel() * t.element_size() // 256) * 256 for t in (g["q"], g["k"], g["v"], g["alpha"],
                                                                      g["b"], g["w"]))
    assert strided == -(-dense // 256) * 256 + copies


def test_backward_from_the_forward_cache_on_strided_inputs():
    c = FWD_CASES[0]
    x, g = inputs(c, seed=303)
    s = strided_inputs(g, c)
    args_d = (g["q"], g["k"], g["v"], g["alpha"])
    args_s = (s["q"], s["k"], s["v"], s["alpha"])
    size = gdn.gdn_chunk_fwd_cache_size(*args_d, h0=g["h0"], **gates(g))
    assert size == gdn.gdn_chunk_fwd_cache_size(*args_s, h0=g["h0"], **gates(s)) and size > 0
    cd = torch.empty(size, dtype=torch.uint8, device="cuda")
    cs = torch.empty(size, dtype=torch.uint8, device="cuda")
    gdn.gdn_chunk_fwd(*args_d, h0=g["h0"], bwd_cache=cd, **gates(g))
    gdn.gdn_chunk_fwd(*args_s, h0=g["h0"], bwd_cache=cs, **gates(s))
    common = dict(h0=g["h0"], grad_o=g["dout"], grad_ht=g["dht"], grads_in_dtype=True)
    gd = gdn.gdn_chunk_bwd(*args_d, fwd_cache=cd, **common, **gates(g))
    gs = gdn.gdn_chunk_bwd(*args_s, fwd_cache=cs, **common, **gates(s))
    torch.cuda.synchronize()
    for key, val in gd.items():
        assert torch.equal(val, gs[key]), key


def test_segment_map_and_no_alloc_forward_on_strided_inputs():
    c = FWD_CASES[0]
    x, g = inputs(c, B=1, T=100, seed=305)
    s = strided_inputs(g, c)
    Md, Nd = gdn.gdn_segment_map(g["q"], g["k"], g["v"], g["alpha"], **gates(g))
    Ms, Ns = gdn.gdn_segment_map(s["q"], s["k"], s["v"], s["alpha"], **gates(s))
    od, _ = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], **gates(g))
    on, _ = gdn.gdn_chunk_fwd_noalloc(s["q"], s["k"], s["v"], s["alpha"], h0=g["h0"], **gates(s))
    torch.cuda.synchronize()
    assert torch.equal(Md, Ms) and torch.equal(Nd, Ns)
    assert torch.equal(od, on)
    assert gdn.gdn_chunk_fwd_noalloc_status() == 0


@pytest.mark.parametrize("gpc", [False, True])
def test_layer_forward_and_backward_on_strided_inputs(gpc):
    B, T, Hk, Hv, d = 1, 130, 1, 2, 128
    x = draw(B, T, Hk, Hv, d, d, alpha_per_channel=gpc, gates_per_channel=gpc, dtype="bf16", gate_dtype="bf16",
             seed=307, has_h0=False, conv=True, swish_gate=True, with_dout=True)
    g = to_cuda(x)
    names = ("q", "k", "v", "alpha", "b", "w", "beta", "z")
    s = fused({n: g.get(n) for n in names if g.get(n) is not None}, offset=2)
    gk = lambda src: dict(beta=src["beta"]) if not gpc else dict(b=src["b"], w=src["w"])
    yd, htd, csd = gdn.gdn_layer_core_fwd(g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"],
                                          want_conv_state=True, **gk(g))
    ys, hts, css = gdn.gdn_layer_core_fwd(s["q"], s["k"], s["v"], g["conv_w"], s["alpha"], s["z"],
                                          want_conv_state=True, **gk(s))
    bd = gdn.gdn_layer_core_bwd(g["q"], g["k"], g["v"], g["conv_w"], g["alpha"], g["z"], g["dout"], **gk(g))
    bs = gdn.gdn_layer_core_bwd(s["q"], s["k"], s["v"], g["conv_w"], s["alpha"], s["z"], g["dout"], **gk(s))
    torch.cuda.synchronize()
    assert torch.equal(yd, ys) and torch.equal(htd, hts) and torch.equal(csd, css)
    for key, val in bd.items():
        if val is not None:
            assert torch.equal(val, bs[key]), key


@pytest.mark.parametrize("conv", [False, True])
def test_decode_reads_strided_inputs_in_place(conv):
    """The decode step's inputs as the t-th token of [N, steps, H, d] tensors (sequence stride
    steps * H * d), against the same step on dense copies."""
    N, steps, Hk, Hv, d = 4, 3, 2, 8, 128
    x = draw(N, steps, Hk, Hv, d, d, alpha_per_channel=True, gates_per_channel=True, dtype="bf16", gate_dtype="bf16",
             seed=309, has_h0=True, conv=conv, swish_gate=True)
    g = to_cuda(x)
    cch = 2 * Hk * d + Hv * d
    hist = torch.randn((N, cch, 3), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).cuda()
    sd, ss = g["h0"].clone(), g["h0"].clone()
    hd, hs = hist.clone(), hist.clone()
    extra = dict(conv_w=g["conv_w"]) if conv else {}
    for t in range(steps):
        view = {n: g[n][:, t] for n in ("q", "k", "v", "alpha", "b", "w", "z")}
        assert not view["q"].is_contiguous()
        dense = {n: v.contiguous() for n, v in view.items()}
        od = gdn.gdn_decode_step(sd, dense["q"], dense["k"], dense["v"], dense["alpha"], b=dense["b"], w=dense["w"],
                                 z=dense["z"], conv_state=hd if conv else None, **extra)
        os_ = gdn.gdn_decode_step(ss, view["q"], view["k"], view["v"], view["alpha"], b=view["b"], w=view["w"],
                                  z=view["z"], conv_state=hs if conv else None, **extra)
        torch.cuda.synchronize()
        assert torch.equal(od, os_) and torch.equal(sd, ss) and torch.equal(hd, hs), t
