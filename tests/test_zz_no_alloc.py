"""gdn_chunk_fwd_noalloc (the forward on the library's built-in scratch array) against
gdn_chunk_fwd with a caller workspace, through the C ABI.

Collected last on purpose: it must pass both in a fresh process (its first call may load the
library's device code) and after every other test has used the library.  Each case runs the
new entry point twice in a row on different inputs, so a second call cannot pass on what the
first one left in the scratch.
"""
import ctypes

import pytest
import torch

from gated_delta_rule_76_b200 import gdn
from gated_delta_rule_76_b200.inputs import draw
from parity import TOL, rel_error

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def gate_kw(g):
    return dict(beta=g["beta"]) if "beta" in g else dict(b=g["b"], w=g["w"])


@pytest.mark.parametrize("case", [
    # tensor-core path: bf16, dk = dv = 128, channel gates, GQA 2 -> 4
    dict(B=2, T=200, Hk=2, Hv=4, d=128, apc=True, gpc=True, dtype="bf16", gdt="bf16", prec="bf16"),
    # CUDA-core path: fp32, d = 64 (its per-chunk factors live in the scratch)
    dict(B=1, T=256, Hk=2, Hv=2, d=64, apc=True, gpc=True, dtype="f32", gdt="f32", prec="f32"),
    # CUDA-core path with scalar gates and a ragged tail
    dict(B=2, T=130, Hk=1, Hv=2, d=64, apc=False, gpc=False, dtype="f32", gdt="f32", prec="f32"),
])
def test_noalloc_matches_workspace_call_twice(case):
    for call, seed in enumerate((31, 32)):
        x = draw(case["B"], case["T"], case["Hk"], case["Hv"], case["d"], case["d"],
                 alpha_per_channel=case["apc"], gates_per_channel=case["gpc"], dtype=case["dtype"],
                 gate_dtype=case["gdt"], seed=seed, has_h0=True)
        g = {k: v.cuda() for k, v in x.items()}
        out_f32 = case["dtype"] == "bf16"
        o_ref, ht_ref = gdn.gdn_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], out_f32=out_f32,
                                          **gate_kw(g))
        o, ht = gdn.gdn_chunk_fwd_noalloc(g["q"], g["k"], g["v"], g["alpha"], h0=g["h0"], out_f32=out_f32,
                                          **gate_kw(g))
        torch.cuda.synchronize()
        tol = TOL[case["prec"]]
        assert rel_error(o, o_ref, case["prec"]) <= tol, f"o, call {call + 1}"
        assert rel_error(ht, ht_ref, case["prec"]) <= tol, f"ht, call {call + 1}"
        # The same kernels on the same inputs, only the scratch differs: the bits agree too.
        assert torch.equal(o, o_ref) and torch.equal(ht, ht_ref), f"bits differ, call {call + 1}"
        # no bounded wait expired: the scratch's status word reads OK
        assert gdn.gdn_chunk_fwd_noalloc_status() == 0, f"status, call {call + 1}"


def test_noalloc_rejects_a_problem_larger_than_its_scratch():
    # fp32 with d = 64 runs on the CUDA-core path, whose per-chunk factors outgrow 16 MiB here.
    B, T, H, d = 1, 8192, 4, 64
    x = draw(B, T, H, H, d, d, alpha_per_channel=True, gates_per_channel=True, dtype="f32",
             gate_dtype="f32", seed=33, has_h0=False)
    g = {k: v.cuda() for k, v in x.items()}
    lib = gdn.load()
    o = torch.empty((B, T, H, d), dtype=torch.float32, device="cuda")
    a, keep = gdn.fwd_args(g["q"], g["k"], g["v"], g["alpha"], g["b"], g["w"], None, None, None, None, 1.0, o,
                           None)
    need = lib.gdn_chunk_fwd_workspace_size(ctypes.byref(a))
    assert need > SCRATCH_BYTES
    before = gdn.kernel_launches()
    status = lib.gdn_chunk_fwd_noalloc(ctypes.byref(a), None)
    assert status == 4  # GDN_ERR_WORKSPACE
    assert "16777216" in lib.gdn_last_error().decode()
    assert gdn.kernel_launches() == before
