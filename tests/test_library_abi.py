"""The C ABI library loads, exports every symbol include/gdn.h declares, its ctypes structs match
the C layouts, and host-side argument validation rejects bad calls before any launch.
Runs without a GPU: no call here reaches a kernel."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest
import torch

from gated_delta_rule_76_b200 import build as gbuild
from gated_delta_rule_76_b200 import gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return gdn.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(gdn.EXPORTED)


def test_selftest_library_exports_its_header(lib):
    text = open(os.path.join(ROOT, "include", "gdn_selftest.h")).read()
    declared = sorted(set(re.findall(r"\b(gdn_selftest_\w+)\s*\(", text)))
    assert declared
    out = subprocess.run(["nm", "-D", "--defined-only", gbuild.SELFTEST_LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (gdn_\w+)", out))
    assert set(declared) <= exported, set(declared) - exported


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", gdn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (gdn_\w+)", out))
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    for f in declared_functions():
        assert hasattr(lib, f)
    assert lib.gdn_version() >= 100


STRUCTS = {"gdn_fwd_args": gdn.FwdArgs, "gdn_bwd_args": gdn.BwdArgs,
           "gdn_decode_args": gdn.DecodeArgs, "gdn_layer_args": gdn.LayerArgs,
           "gdn_layer_bwd_args": gdn.LayerBwdArgs, "gdn_strides": gdn.Strides}


def test_ctypes_structs_match_c_layout():
    """Compile a host program that prints sizeof/offsetof of every field of every struct."""
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "gdn.h"', "int main(void) {"]
    for cname, py in STRUCTS.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines.append("return 0; }")
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        open(src, "w").write("\n".join(lines))
        subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), src, "-o", exe])
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {}
    for line in out:
        if line.strip():
            parts = line.split()
            got[(parts[0], parts[1])] = int(parts[2])
    for cname, py in STRUCTS.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


def _fwd(**kw):
    base = dict(q=16, k=32, v=48, alpha=64, b=80, w=96, h0=None, z=None, o=1 << 20, ht=None,
                head_map=None, B=1, T=64, Hk=1, Hv=1, dk=64, dv=64, scale=1.0,
                alpha_per_channel=1, gates_per_channel=1, dtype=0, gate_dtype=0)
    base.update(kw)
    return gdn.FwdArgs(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(dk=96, dv=96), 2),                  # unsupported head size
    (dict(dk=64, dv=128), 2),                 # dk != dv
    (dict(Hk=3, Hv=4), 1),                    # Hv not a multiple of Hk without a map
    (dict(B=0), 1),
    (dict(q=None), 1),                        # missing input
    (dict(w=None), 1),                        # channel gates without w
    (dict(gates_per_channel=0), 1),           # scalar gates but w given
    (dict(dtype=1, gate_dtype=0), 2),         # fp32 tensors with bf16 gates
    (dict(q=18), 1),                          # misaligned
    (dict(o=32), 1),                          # output overlaps an input
    (dict(dtype=7), 1),
])
def test_host_validation_rejects_before_launch(lib, kw, code):
    a = _fwd(**kw)
    ws = ctypes.c_void_p(1 << 30)
    rc = lib.gdn_chunk_fwd(ctypes.byref(a), ws, 1 << 30, None)
    assert rc == code, lib.gdn_last_error()
    assert lib.gdn_last_error().decode()


def test_workspace_checks(lib):
    a = _fwd()
    need = lib.gdn_chunk_fwd_workspace_size(ctypes.byref(a))
    assert need > 0
    assert lib.gdn_chunk_fwd(ctypes.byref(a), None, 0, None) == 4
    assert lib.gdn_chunk_fwd(ctypes.byref(a), ctypes.c_void_p(1 << 30), need - 1, None) == 4
    assert lib.gdn_chunk_fwd(ctypes.byref(a), ctypes.c_void_p((1 << 30) + 16), need, None) == 4
    assert lib.gdn_chunk_fwd(None, None, 0, None) == 1


def test_workspace_size_scales_with_chunks(lib):
    small = lib.gdn_chunk_fwd_workspace_size(ctypes.byref(_fwd(T=64)))
    big = lib.gdn_chunk_fwd_workspace_size(ctypes.byref(_fwd(T=65)))
    assert big > small  # a ragged tail adds a chunk
    assert lib.gdn_chunk_fwd_workspace_size(None) == 0


def test_forward_cache_validation_on_the_host(lib):
    # fp32 tensors run on the CUDA-core path, which keeps no cache: size 0, a cache is refused
    a = _fwd(dtype=1, gate_dtype=1)
    assert lib.gdn_chunk_fwd_cache_size(ctypes.byref(a)) == 0
    a = _fwd(dtype=1, gate_dtype=1, bwd_cache=1 << 24, bwd_cache_bytes=1 << 20)
    rc = lib.gdn_chunk_fwd(ctypes.byref(a), ctypes.c_void_p(1 << 30), 1 << 30, None)
    assert rc == 2, lib.gdn_last_error()
    # a cache must start on a 256-byte boundary and may not overlap an output
    a = _fwd(bwd_cache=(1 << 24) + 16, bwd_cache_bytes=1 << 20)
    assert lib.gdn_chunk_fwd(ctypes.byref(a), ctypes.c_void_p(1 << 30), 1 << 30, None) == 1
    a = _fwd(bwd_cache=1 << 20, bwd_cache_bytes=1 << 20)
    assert lib.gdn_chunk_fwd(ctypes.byref(a), ctypes.c_void_p(1 << 30), 1 << 30, None) == 1


def _layer_bwd(**kw):
    M = 1 << 16
    base = dict(xq=16, xk=32, xv=48, conv_w=64, alpha=80, b=96, w=None, z=112, h0=None, head_map=None,
                grad_y=128, grad_ht=None, grad_xq=16 * M, grad_xk=17 * M, grad_xv=18 * M, grad_conv_w=19 * M,
                grad_alpha=20 * M, grad_b=21 * M, grad_w=None, grad_z=22 * M, grad_h0=None,
                B=1, T=64, Hk=1, Hv=1, dk=64, dv=64, scale=1.0, alpha_per_channel=0, gates_per_channel=0,
                dtype=0, gate_dtype=1)
    base.update(kw)
    return gdn.LayerBwdArgs(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(dk=64, dv=128), 2),                 # the layer needs dk == dv
    (dict(grad_y=None), 1),                   # missing gradient of y
    (dict(grad_conv_w=None), 1),              # missing output
    (dict(grad_w=23 << 16), 1),               # scalar gates but grad_w given
    (dict(gates_per_channel=1, alpha_per_channel=1), 1),  # channel gates without w / grad_w
    (dict(grad_xq=16), 1),                    # output overlaps an input
    (dict(grad_z=(22 << 16) + 8), 1),         # misaligned output
])
def test_layer_backward_host_validation(lib, kw, code):
    a = _layer_bwd(**kw)
    rc = lib.gdn_layer_core_bwd(ctypes.byref(a), ctypes.c_void_p(1 << 34), 1 << 34, None)
    assert rc == code, lib.gdn_last_error()
    assert lib.gdn_last_error().decode()


def _layer_fwd(**kw):
    M = 1 << 16
    base = dict(xq=16, xk=32, xv=48, conv_w=64, alpha=80, b=96, w=None, z=112, h0=None, y=16 * M, ht=None,
                conv_state_out=None, head_map=None, B=1, T=64, Hk=1, Hv=1, dk=128, dv=128, scale=1.0,
                alpha_per_channel=0, gates_per_channel=0, dtype=0, gate_dtype=1, out_f32=0, bwd_cache=None,
                bwd_cache_bytes=0)
    base.update(kw)
    return gdn.LayerArgs(**base)


def test_layer_forward_cache_on_the_host(lib):
    """Only the tensor-core form (bf16, d = 128, scalar gates, no h0) keeps a layer cache; a cache
    elsewhere, misaligned, overlapping an output or too small is refused before any launch."""
    size = lambda **kw: lib.gdn_layer_core_fwd_cache_size(ctypes.byref(_layer_fwd(**kw)))
    need = size()
    assert need > 0 and size(T=65) > need
    assert size(h0=144) == 0 and size(dtype=1) == 0 and size(dk=64, dv=64) == 0
    assert size(alpha_per_channel=1, gates_per_channel=1, w=128, gate_dtype=0) == 0
    ws = ctypes.c_void_p(1 << 34)
    run = lambda **kw: lib.gdn_layer_core_fwd(ctypes.byref(_layer_fwd(**kw)), ws, 1 << 34, None)
    assert run(h0=144, bwd_cache=1 << 30, bwd_cache_bytes=need) == 2
    assert run(bwd_cache=(1 << 30) + 16, bwd_cache_bytes=need) == 1
    assert run(bwd_cache=16 << 16, bwd_cache_bytes=need) == 1      # overlaps y
    assert run(bwd_cache=1 << 30, bwd_cache_bytes=need - 1) == 4
    bwd = lambda **kw: lib.gdn_layer_core_bwd(ctypes.byref(_layer_bwd(dk=128, dv=128, **kw)), ws, 1 << 34, None)
    assert bwd(h0=144, fwd_cache=1 << 30, fwd_cache_bytes=need) == 2
    assert bwd(fwd_cache=(1 << 30) + 16, fwd_cache_bytes=need) == 1
    assert bwd(fwd_cache=1 << 30, fwd_cache_bytes=need - 1) == 1
    # with a cache the backward's workspace leaves out the conv results, o, the states and V'
    wsz = lambda **kw: lib.gdn_layer_core_bwd_workspace_size(ctypes.byref(_layer_bwd(dk=128, dv=128, T=4096, **kw)))
    assert 0 < wsz(fwd_cache=1 << 30, fwd_cache_bytes=1 << 40) < wsz()


def test_layer_backward_workspace_forms(lib):
    """bf16, d = 128, scalar gates and no h0 take the tensor-core form, whose workspace (states, V',
    two sets of recurrence gradients) is smaller than the CUDA-core form's per-chunk factors; an h0,
    fp32 tensors or d = 64 take the CUDA-core form."""
    size = lambda **kw: lib.gdn_layer_core_bwd_workspace_size(ctypes.byref(_layer_bwd(T=4096, **kw)))
    tc = size(dk=128, dv=128)
    assert 0 < tc < size(dk=128, dv=128, h0=144)
    assert tc < size(dk=128, dv=128, dtype=1)


def test_layer_backward_workspace(lib):
    a = _layer_bwd()
    need = lib.gdn_layer_core_bwd_workspace_size(ctypes.byref(a))
    assert need > 0
    assert lib.gdn_layer_core_bwd_workspace_size(ctypes.byref(_layer_bwd(T=65))) > need
    assert lib.gdn_layer_core_bwd(ctypes.byref(a), ctypes.c_void_p(1 << 34), need - 1, None) == 4
    assert lib.gdn_layer_core_bwd(None, None, 0, None) == 1


def test_binding_checks_a_host_head_map():
    """Entries outside [0, Hk) are refused before the map is uploaded (the kernels only clamp)."""
    from gated_delta_rule_76_b200 import gdn
    assert gdn._head_map([0, 1, 1, 0], "cpu", 2).tolist() == [0, 1, 1, 0]
    for bad in ([0, 2], [-1, 0]):
        with pytest.raises(gdn.GdnError):
            gdn._head_map(bad, "cpu", 2)


def test_segment_map_and_compose_host_validation(lib):
    """gdn_segment_map takes no h0 and needs ht (N) and M; gdn_state_compose checks its sizes and
    overlaps.  Rejected on the host, before any launch (fake device addresses, never touched)."""
    P = ctypes.c_void_p
    M, N = P(1 << 24), P(1 << 25)
    before = gdn.kernel_launches()
    a = _fwd(o=None, ht=1 << 25, h0=1 << 26)
    assert lib.gdn_segment_map(ctypes.byref(a), M, P(1 << 30), 1 << 30, None) == 1  # h0 given
    a = _fwd(o=None, ht=None)
    assert lib.gdn_segment_map(ctypes.byref(a), M, P(1 << 30), 1 << 30, None) == 1  # no ht
    a = _fwd(o=None, ht=1 << 25)
    assert lib.gdn_segment_map(ctypes.byref(a), None, P(1 << 30), 1 << 30, None) == 1  # no M
    a = _fwd(o=None, ht=1 << 24)
    assert lib.gdn_segment_map(ctypes.byref(a), M, P(1 << 30), 1 << 30, None) == 1  # M overlaps ht
    a = _fwd(o=None, ht=1 << 25)
    assert lib.gdn_segment_map(ctypes.byref(a), M, None, 0, None) == 4  # no workspace
    assert lib.gdn_state_compose(M, None, None, N, 1, 32, 32, 0, None) == 2
    assert lib.gdn_state_compose(None, None, None, N, 1, 128, 128, 0, None) == 1
    assert lib.gdn_state_compose(M, None, None, M, 1, 128, 128, 0, None) == 1  # output overlaps M
    assert lib.gdn_state_compose(M, None, None, N, 1, 64, 128, 1, None) == 1   # M^T needs dk == dv
    assert gdn.kernel_launches() == before


def test_gate_logit_arguments_rejected_on_the_host(lib):
    """gate_logits needs alpha_scale; alpha_scale without gate_logits, or a flag other than 0/1, is
    an error; nothing is launched."""
    before = gdn.kernel_launches()
    ws = ctypes.c_void_p(1 << 30)
    for kw in (dict(gate_logits=1), dict(alpha_scale=1 << 27), dict(gate_logits=2, alpha_scale=1 << 27)):
        a = _fwd(**kw)
        assert lib.gdn_chunk_fwd(ctypes.byref(a), ws, 1 << 30, None) == 1, kw
        assert "gate_logits" in lib.gdn_last_error().decode() or "alpha_scale" in lib.gdn_last_error().decode()
    assert gdn.kernel_launches() == before


def _bwd(**kw):
    base = dict(q=16, k=32, v=48, alpha=64, b=80, w=96, h0=None, head_map=None, grad_o=112, grad_ht=None,
                grad_q=1 << 20, grad_k=2 << 20, grad_v=3 << 20, grad_alpha=4 << 20, grad_b=5 << 20,
                grad_w=6 << 20, grad_h0=None, B=1, T=64, Hk=1, Hv=1, dk=64, dv=64, scale=1.0,
                alpha_per_channel=1, gates_per_channel=1, dtype=0, gate_dtype=0)
    base.update(kw)
    return gdn.BwdArgs(**base)


def test_gradient_dtype_option_on_the_host(lib):
    """grads_in_dtype is 0 or 1; bf16 gradients of a bf16 problem the tensor-core backward does not
    serve (here dk = 64) are refused as unsupported; nothing is launched (fake device addresses)."""
    before = gdn.kernel_launches()
    ws = ctypes.c_void_p(1 << 30)
    a = _bwd(grads_in_dtype=2)
    assert lib.gdn_chunk_bwd(ctypes.byref(a), ws, 1 << 30, None) == 1
    assert "grads_in_dtype" in lib.gdn_last_error().decode()
    a = _bwd(grads_in_dtype=1)
    assert lib.gdn_chunk_bwd(ctypes.byref(a), ws, 1 << 30, None) == 2
    assert "grads_in_dtype" in lib.gdn_last_error().decode()
    # bf16 gradients take half the bytes: outputs that overlap as fp32 are disjoint as bf16 (the
    # call then stops at the unsupported path, after the buffer checks)
    close = dict(grad_k=(1 << 20) + 64 * 64 * 2)
    a = _bwd(**close)
    assert lib.gdn_chunk_bwd(ctypes.byref(a), ws, 1 << 30, None) == 1
    assert "overlap" in lib.gdn_last_error().decode()
    a = _bwd(grads_in_dtype=1, **close)
    assert lib.gdn_chunk_bwd(ctypes.byref(a), ws, 1 << 30, None) == 2
    assert gdn.kernel_launches() == before


def test_token_strides_on_the_host(lib):
    """gdn_strides: a stride below a token's element count (or above 2^31) is refused; a strided
    input needs only its element alignment and adds its dense copy to the workspace; an output
    inside a strided input's span overlaps it; the backward refuses a z stride.  Fake device
    addresses: every call here stops before a launch."""
    before = gdn.kernel_launches()
    ws = ctypes.c_void_p(1 << 30)
    row = 64  # Hk * dk of _fwd()
    a = _fwd()
    a.strides.q = row - 1
    assert lib.gdn_chunk_fwd(ctypes.byref(a), ws, 1 << 30, None) == 1
    assert "token stride of q" in lib.gdn_last_error().decode()
    a.strides.q = (1 << 31) + 1
    assert lib.gdn_chunk_fwd(ctypes.byref(a), ws, 1 << 30, None) == 1
    # dense stride given explicitly: same workspace as 0
    dense = lib.gdn_chunk_fwd_workspace_size(ctypes.byref(_fwd()))
    a = _fwd()
    a.strides.q = row
    assert lib.gdn_chunk_fwd_workspace_size(ctypes.byref(a)) == dense
    # a strided q (2-byte aligned, 3 * row apart) and a strided alpha: their dense copies
    a = _fwd(q=18, o=1 << 22)
    a.strides.q = 3 * row
    a.strides.alpha = 2 * row
    need = lib.gdn_chunk_fwd_workspace_size(ctypes.byref(a))
    copy = 64 * row * 2  # 64 tokens of 64 bf16 values, a multiple of 256 bytes
    assert need == (dense + 255) // 256 * 256 + 2 * copy
    # accepted by the buffer checks (a dense q at 18 is not), then stopped by a short workspace
    assert lib.gdn_chunk_fwd(ctypes.byref(a), ws, need - 1, None) == 4
    assert lib.gdn_chunk_fwd(ctypes.byref(_fwd(q=18)), ws, 1 << 30, None) == 1
    # o placed inside q's span (3 * row * 63 + row elements from 18) overlaps it
    a = _fwd(q=1 << 20, o=(1 << 20) + 2 * 64 * row * 2)
    a.strides.q = 3 * row
    assert lib.gdn_chunk_fwd(ctypes.byref(a), ws, 1 << 30, None) == 1
    assert "overlap" in lib.gdn_last_error().decode()
    # the backward takes no z
    b = _bwd()
    b.strides.z = 64
    assert lib.gdn_chunk_bwd(ctypes.byref(b), ws, 1 << 30, None) == 1
    assert "strides.z" in lib.gdn_last_error().decode()
    b = _bwd()
    b.strides.v = 63
    assert lib.gdn_chunk_bwd(ctypes.byref(b), ws, 1 << 30, None) == 1
    assert gdn.kernel_launches() == before


def test_binding_token_strides():
    """The binding's token stride of a view (CPU tensors: the rule only, nothing is called)."""
    buf = torch.zeros((2 * 5, 200))
    v = buf[:, 64:128].view(2, 5, 1, 64)  # a slice of a fused projection buffer
    assert gdn._token_stride(v.shape, v.stride(), 2) == 200
    d = torch.zeros((2, 5, 2, 64))
    assert gdn._token_stride(d.shape, d.stride(), 2) == 0
    one = buf[:5, 0:64].view(1, 5, 1, 64)  # B = 1: the T stride alone
    assert gdn._token_stride(one.shape, one.stride(), 2) == 200
    tok = buf[:1, 0:128].view(1, 1, 2, 64)  # a single token: dense
    assert gdn._token_stride(tok.shape, tok.stride(), 2) == 0
    dec = buf[:, 64:128].view(10, 1, 64)  # decode: [N, H, d]
    assert gdn._token_stride(dec.shape, dec.stride(), 1) == 200
    with pytest.raises(gdn.GdnError, match="heads and channels are dense"):
        x = d[:, :, :, :32]
        gdn._token_stride(x.shape, x.stride(), 2)
    with pytest.raises(gdn.GdnError, match="evenly spaced"):
        x = torch.zeros((2, 7, 64))[:, :5]
        gdn._token_stride(x.shape, x.stride(), 2)
    with pytest.raises(gdn.GdnError, match="CUDA tensors only"):
        gdn._tok(v)


def test_token_strides_on_every_call(lib):
    """Stride validation and the dense copies' workspace on the segment map, the decode step and
    both layer calls (fake device addresses; every call stops on the host)."""
    before = gdn.kernel_launches()
    P = ctypes.c_void_p
    ws = P(1 << 34)
    # segment map: a k stride below the token's 64 elements
    a = _fwd(o=None, ht=1 << 25)
    a.strides.k = 63
    assert lib.gdn_segment_map(ctypes.byref(a), P(1 << 24), ws, 1 << 34, None) == 1
    assert "token stride of k" in lib.gdn_last_error().decode()
    a = _fwd(o=None, ht=1 << 25)
    dense = lib.gdn_segment_map_workspace_size(ctypes.byref(a))
    a.strides.q = 128
    assert lib.gdn_segment_map_workspace_size(ctypes.byref(a)) == (dense + 255) // 256 * 256 + 64 * 64 * 2
    # decode: strides are read in place, so only the bounds are checked
    d = gdn.DecodeArgs(q=16, k=32, v=48, alpha=64, b=80, w=96, state=1 << 20, o=1 << 21, N=2, Hk=1, Hv=1, dk=64,
                       dv=64, scale=1.0, alpha_per_channel=1, gates_per_channel=1, dtype=0, gate_dtype=0)
    d.strides.v = 10
    assert lib.gdn_decode_step(ctypes.byref(d), None) == 1
    assert "token stride of v" in lib.gdn_last_error().decode()
    d.strides.v = 0
    d.strides.z = (1 << 31) + 1
    assert lib.gdn_decode_step(ctypes.byref(d), None) == 1
    # layer forward: z below its 128 elements; a strided xq adds its copy and needs its element alignment only
    f = _layer_fwd()
    f.strides.z = 127
    assert lib.gdn_layer_core_fwd(ctypes.byref(f), ws, 1 << 34, None) == 1
    assert "token stride of z" in lib.gdn_last_error().decode()
    dense = lib.gdn_layer_core_fwd_workspace_size(ctypes.byref(_layer_fwd()))
    f = _layer_fwd(xq=18)
    assert lib.gdn_layer_core_fwd(ctypes.byref(f), ws, 1 << 34, None) == 1  # dense xq at 18: misaligned
    f.strides.q = 256
    need = lib.gdn_layer_core_fwd_workspace_size(ctypes.byref(f))
    assert need == (dense + 255) // 256 * 256 + 64 * 128 * 2
    assert lib.gdn_layer_core_fwd(ctypes.byref(f), ws, need - 1, None) == 4
    # layer backward: a negative stride, then a strided alpha's copy in the workspace
    g = _layer_bwd()
    g.strides.b = -1
    assert lib.gdn_layer_core_bwd(ctypes.byref(g), ws, 1 << 34, None) == 1
    dense = lib.gdn_layer_core_bwd_workspace_size(ctypes.byref(_layer_bwd()))
    g = _layer_bwd()
    g.strides.alpha = 4  # scalar alpha: 1 element a token
    assert lib.gdn_layer_core_bwd_workspace_size(ctypes.byref(g)) == (dense + 255) // 256 * 256 + 256
    assert gdn.kernel_launches() == before
