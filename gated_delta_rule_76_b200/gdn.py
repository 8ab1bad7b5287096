"""Thin Python binding of libgdn (include/gdn.h), same names as the C ABI.

Only argument marshalling lives here: torch allocates device memory (outputs and the
workspace) and provides the stream; every step of the recurrence runs in the CUDA kernels of
libgdn.so.  There is no CPU fallback: if the library is missing or a tensor is not on a CUDA
device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_BF16, GDN_F32 = 0, 1
_STATUS = {0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_UNSUPPORTED", 3: "GDN_ERR_CUDA",
           4: "GDN_ERR_WORKSPACE", 5: "GDN_ERR_TIMEOUT"}

P = ctypes.c_void_p
I64 = ctypes.c_int64
I32 = ctypes.c_int32
F32 = ctypes.c_float


class Strides(ctypes.Structure):
    """gdn_strides: token strides in elements (0 = dense)."""
    _fields_ = [("q", I64), ("k", I64), ("v", I64), ("alpha", I64), ("b", I64), ("w", I64), ("z", I64)]


class FwdArgs(ctypes.Structure):
    _fields_ = [("q", P), ("k", P), ("v", P), ("alpha", P), ("b", P), ("w", P), ("h0", P),
                ("z", P), ("o", P), ("ht", P), ("head_map", P),
                ("B", I64), ("T", I64), ("Hk", I64), ("Hv", I64), ("dk", I64), ("dv", I64),
                ("scale", F32), ("alpha_per_channel", I32), ("gates_per_channel", I32),
                ("dtype", I32), ("gate_dtype", I32), ("out_f32", I32),
                ("bwd_cache", P), ("bwd_cache_bytes", ctypes.c_size_t), ("gate_logits", I32),
                ("alpha_scale", P), ("strides", Strides)]


class BwdArgs(ctypes.Structure):
    _fields_ = [("q", P), ("k", P), ("v", P), ("alpha", P), ("b", P), ("w", P), ("h0", P),
                ("head_map", P), ("grad_o", P), ("grad_ht", P), ("grad_q", P), ("grad_k", P),
                ("grad_v", P), ("grad_alpha", P), ("grad_b", P), ("grad_w", P), ("grad_h0", P),
                ("B", I64), ("T", I64), ("Hk", I64), ("Hv", I64), ("dk", I64), ("dv", I64),
                ("scale", F32), ("alpha_per_channel", I32), ("gates_per_channel", I32),
                ("dtype", I32), ("gate_dtype", I32),
                ("fwd_cache", P), ("fwd_cache_bytes", ctypes.c_size_t), ("gate_logits", I32),
                ("alpha_scale", P), ("grad_alpha_scale", P), ("grads_in_dtype", I32), ("strides", Strides)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("q", P), ("k", P), ("v", P), ("alpha", P), ("b", P), ("w", P), ("state", P),
                ("o", P), ("head_map", P), ("conv_state", P), ("conv_w", P), ("z", P),
                ("N", I64), ("Hk", I64), ("Hv", I64), ("dk", I64), ("dv", I64),
                ("scale", F32), ("alpha_per_channel", I32), ("gates_per_channel", I32),
                ("dtype", I32), ("gate_dtype", I32), ("out_f32", I32), ("gate_logits", I32),
                ("alpha_scale", P), ("strides", Strides)]


class LayerArgs(ctypes.Structure):
    _fields_ = [("xq", P), ("xk", P), ("xv", P), ("conv_w", P), ("alpha", P), ("b", P), ("w", P),
                ("z", P), ("h0", P), ("y", P), ("ht", P), ("conv_state_out", P), ("head_map", P),
                ("B", I64), ("T", I64), ("Hk", I64), ("Hv", I64), ("dk", I64), ("dv", I64),
                ("scale", F32), ("alpha_per_channel", I32), ("gates_per_channel", I32),
                ("dtype", I32), ("gate_dtype", I32), ("out_f32", I32), ("bwd_cache", P),
                ("bwd_cache_bytes", ctypes.c_size_t), ("norm_w", P), ("norm_eps", F32), ("gate_logits", I32),
                ("alpha_scale", P), ("strides", Strides)]


class LayerBwdArgs(ctypes.Structure):
    _fields_ = [("xq", P), ("xk", P), ("xv", P), ("conv_w", P), ("alpha", P), ("b", P), ("w", P),
                ("z", P), ("h0", P), ("head_map", P), ("grad_y", P), ("grad_ht", P),
                ("grad_xq", P), ("grad_xk", P), ("grad_xv", P), ("grad_conv_w", P), ("grad_alpha", P),
                ("grad_b", P), ("grad_w", P), ("grad_z", P), ("grad_h0", P),
                ("B", I64), ("T", I64), ("Hk", I64), ("Hv", I64), ("dk", I64), ("dv", I64),
                ("scale", F32), ("alpha_per_channel", I32), ("gates_per_channel", I32),
                ("dtype", I32), ("gate_dtype", I32), ("fwd_cache", P), ("fwd_cache_bytes", ctypes.c_size_t),
                ("norm_w", P), ("norm_eps", F32), ("grad_norm_w", P), ("gate_logits", I32),
                ("alpha_scale", P), ("grad_alpha_scale", P), ("strides", Strides)]


EXPORTED = ["gdn_chunk_fwd_cache_size", "gdn_chunk_fwd_workspace_size", "gdn_chunk_fwd", "gdn_chunk_fwd_noalloc",
            "gdn_chunk_fwd_noalloc_status", "gdn_chunk_bwd_workspace_size",
            "gdn_chunk_bwd", "gdn_decode_step", "gdn_layer_core_fwd_cache_size", "gdn_layer_core_fwd_workspace_size",
            "gdn_layer_core_fwd", "gdn_layer_core_bwd_workspace_size", "gdn_layer_core_bwd",
            "gdn_segment_map_workspace_size", "gdn_segment_map", "gdn_state_compose",
            "gdn_workspace_status", "gdn_last_error", "gdn_kernel_launches", "gdn_version"]

_lib = None


class GdnError(RuntimeError):
    pass


def load(path: str = LIB_PATH):
    """Load libgdn.so and declare its C signatures.  Raises if the library is missing."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise GdnError(f"{path} is missing: build it with `python -m gated_delta_rule_76_b200.build`")
    lib = ctypes.CDLL(path)
    lib.gdn_chunk_fwd_cache_size.argtypes = [ctypes.POINTER(FwdArgs)]
    lib.gdn_chunk_fwd_cache_size.restype = ctypes.c_size_t
    lib.gdn_chunk_fwd_workspace_size.argtypes = [ctypes.POINTER(FwdArgs)]
    lib.gdn_chunk_fwd_workspace_size.restype = ctypes.c_size_t
    lib.gdn_chunk_fwd.argtypes = [ctypes.POINTER(FwdArgs), P, ctypes.c_size_t, P]
    lib.gdn_chunk_fwd.restype = ctypes.c_int
    lib.gdn_chunk_fwd_noalloc.argtypes = [ctypes.POINTER(FwdArgs), P]
    lib.gdn_chunk_fwd_noalloc.restype = ctypes.c_int
    lib.gdn_chunk_fwd_noalloc_status.argtypes = [P]
    lib.gdn_chunk_fwd_noalloc_status.restype = ctypes.c_int
    lib.gdn_chunk_bwd_workspace_size.argtypes = [ctypes.POINTER(BwdArgs)]
    lib.gdn_chunk_bwd_workspace_size.restype = ctypes.c_size_t
    lib.gdn_chunk_bwd.argtypes = [ctypes.POINTER(BwdArgs), P, ctypes.c_size_t, P]
    lib.gdn_chunk_bwd.restype = ctypes.c_int
    lib.gdn_decode_step.argtypes = [ctypes.POINTER(DecodeArgs), P]
    lib.gdn_decode_step.restype = ctypes.c_int
    lib.gdn_layer_core_fwd_cache_size.argtypes = [ctypes.POINTER(LayerArgs)]
    lib.gdn_layer_core_fwd_cache_size.restype = ctypes.c_size_t
    lib.gdn_layer_core_fwd_workspace_size.argtypes = [ctypes.POINTER(LayerArgs)]
    lib.gdn_layer_core_fwd_workspace_size.restype = ctypes.c_size_t
    lib.gdn_layer_core_fwd.argtypes = [ctypes.POINTER(LayerArgs), P, ctypes.c_size_t, P]
    lib.gdn_layer_core_fwd.restype = ctypes.c_int
    lib.gdn_layer_core_bwd_workspace_size.argtypes = [ctypes.POINTER(LayerBwdArgs)]
    lib.gdn_layer_core_bwd_workspace_size.restype = ctypes.c_size_t
    lib.gdn_layer_core_bwd.argtypes = [ctypes.POINTER(LayerBwdArgs), P, ctypes.c_size_t, P]
    lib.gdn_layer_core_bwd.restype = ctypes.c_int
    lib.gdn_segment_map_workspace_size.argtypes = [ctypes.POINTER(FwdArgs)]
    lib.gdn_segment_map_workspace_size.restype = ctypes.c_size_t
    lib.gdn_segment_map.argtypes = [ctypes.POINTER(FwdArgs), P, P, ctypes.c_size_t, P]
    lib.gdn_segment_map.restype = ctypes.c_int
    lib.gdn_state_compose.argtypes = [P, P, P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, P]
    lib.gdn_state_compose.restype = ctypes.c_int
    lib.gdn_workspace_status.argtypes = [P, P]
    lib.gdn_workspace_status.restype = ctypes.c_int
    lib.gdn_last_error.argtypes = []
    lib.gdn_last_error.restype = ctypes.c_char_p
    lib.gdn_kernel_launches.argtypes = []
    lib.gdn_kernel_launches.restype = ctypes.c_longlong
    lib.gdn_version.argtypes = []
    lib.gdn_version.restype = ctypes.c_int
    if path == LIB_PATH:
        _lib = lib
    return lib


def kernel_launches() -> int:
    """Kernels launched by libgdn in this process so far."""
    return int(load().gdn_kernel_launches())


def check(status: int, what: str):
    if status != 0:
        msg = load().gdn_last_error().decode(errors="replace")
        raise GdnError(f"{what}: {_STATUS.get(status, status)}: {msg}")


# ---------------------------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------------------------
def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise GdnError("libgdn takes CUDA tensors only (there is no CPU path)")
    if not t.is_contiguous():
        raise GdnError("libgdn takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _tok(t: Optional[torch.Tensor], lead: int = 2):
    """A token-major input as (pointer, token stride in elements, 0 when dense).  Besides a
    contiguous tensor it takes a view whose heads and channels are dense and whose tokens are
    evenly spaced, such as a slice of a fused projection [B, T, C] viewed as [B, T, H, d].
    ``lead`` is the number of token dimensions (2: [B, T, ...]; 1: the decode step's [N, ...])."""
    if t is None:
        return None, 0
    if t.is_contiguous():
        return _ptr(t), 0
    if not t.is_cuda:
        raise GdnError("libgdn takes CUDA tensors only (there is no CPU path)")
    return ctypes.c_void_p(t.data_ptr()), _token_stride(tuple(t.shape), tuple(t.stride()), lead)


def _token_stride(shape, strides, lead: int) -> int:
    """The token stride, in elements, of a tensor of this shape and these strides (0 when its
    tokens are dense); its first ``lead`` dimensions index tokens."""
    row = 1
    for dim in range(len(shape) - 1, lead - 1, -1):
        if shape[dim] != 1 and strides[dim] != row:
            raise GdnError("libgdn takes token-major tensors whose heads and channels are dense")
        row *= shape[dim]
    dims = [d for d in range(lead) if shape[d] != 1]
    s = strides[dims[-1]] if dims else row
    if len(dims) == 2 and strides[dims[0]] != shape[dims[1]] * s:
        raise GdnError("libgdn takes token-major tensors whose tokens are evenly spaced")
    if s < row:
        raise GdnError(f"token stride {s} is below the {row} elements of a token")
    return 0 if s == row else s


def _inputs(lead: int, q, k, v, alpha, b, w, z=None):
    """Pointers and gdn_strides of a call's token-major inputs."""
    ptrs, strides = {}, {}
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("b", b), ("w", w), ("z", z)):
        ptrs[name], strides[name] = _tok(t, lead)
    return ptrs, Strides(**strides)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise GdnError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return None
    if workspace is not None and workspace.numel() * workspace.element_size() >= nbytes:
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _gates(alpha, b, w, beta):
    if beta is not None:
        if b is not None or w is not None:
            raise GdnError("give either beta or (b, w)")
        return beta, None, 0
    if b is None or w is None:
        raise GdnError("channel gates need both b and w")
    return b, w, 1


def _head_map(head_map, device, Hk: int):
    """The value-head -> key-head map as an int32 device array.  A map given on the host (a list
    or a CPU tensor) is checked before it is uploaded: every entry must be in [0, Hk).  A map
    already on the device is passed through unchecked (checking it would synchronise)."""
    if head_map is None:
        return None
    if not torch.is_tensor(head_map):
        head_map = torch.tensor(head_map, dtype=torch.int32)
    if head_map.device.type == "cpu" and head_map.numel():
        lo, hi = int(head_map.min()), int(head_map.max())
        if lo < 0 or hi >= Hk:
            raise GdnError(f"head_map entries must be in [0, {Hk}); got [{lo}, {hi}]")
    return head_map.to(device=device, dtype=torch.int32).contiguous()


# ---------------------------------------------------------------------------------------------
# public calls
#
# Token-major inputs (q, k, v, the gates, z; xq, xk, xv for the layer calls) may be views whose
# tokens are evenly spaced and whose heads and channels are dense, such as column slices of one
# fused projection buffer viewed as [B, T, H, d]: they are passed with their token stride
# (gdn_strides), without a copy here.  Every other tensor must be contiguous.
# ---------------------------------------------------------------------------------------------
def fwd_args(q, k, v, alpha, b=None, w=None, beta=None, h0=None, z=None, head_map=None,
             scale: float = 1.0, o=None, ht=None, bwd_cache=None, alpha_scale=None) -> Tuple[FwdArgs, list]:
    """Build the gdn_fwd_args struct (the returned list keeps referenced tensors alive).
    ``alpha_scale`` [Hv] fp32: the gates are logits (alpha = exp(-alpha_scale softplus(x)),
    b, w, beta = sigmoid(x))."""
    bb, ww, gpc = _gates(alpha, b, w, beta)
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    hm = _head_map(head_map, q.device, q.shape[-2])
    tp, ts = _inputs(2, q, k, v, alpha, bb, ww, z)
    a = FwdArgs(q=tp["q"], k=tp["k"], v=tp["v"], alpha=tp["alpha"], b=tp["b"], w=tp["w"],
                h0=_ptr(h0), z=tp["z"], o=_ptr(o), ht=_ptr(ht), head_map=_ptr(hm),
                B=B, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv, scale=scale,
                alpha_per_channel=int(alpha.dim() == 4), gates_per_channel=gpc,
                dtype=_dt(q), gate_dtype=_dt(alpha),
                out_f32=int(o is not None and o.dtype == torch.float32 and q.dtype != torch.float32),
                bwd_cache=_ptr(bwd_cache),
                bwd_cache_bytes=0 if bwd_cache is None else bwd_cache.numel() * bwd_cache.element_size(),
                gate_logits=int(alpha_scale is not None), alpha_scale=_ptr(alpha_scale), strides=ts)
    return a, [q, k, v, alpha, bb, ww, h0, z, o, ht, hm, bwd_cache, alpha_scale]


def gdn_chunk_fwd_cache_size(q, k, v, alpha, b=None, w=None, beta=None, h0=None, head_map=None,
                             scale: float = 1.0, alpha_scale=None) -> int:
    """Bytes of the forward cache gdn_chunk_fwd(..., bwd_cache=) can fill for a later backward
    (0: this problem runs on the CUDA-core path, which keeps none)."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    a, keep = fwd_args(q, k, v, alpha, b, w, beta, h0, None, head_map, scale, alpha_scale=alpha_scale)
    return int(load().gdn_chunk_fwd_cache_size(ctypes.byref(a)))


def gdn_chunk_fwd(q, k, v, alpha, b=None, w=None, beta=None, h0=None, z=None, head_map=None,
                  scale: float = 1.0, *, o=None, ht=None, want_ht: bool = True, out_f32: bool = False,
                  bwd_cache: Optional[torch.Tensor] = None, alpha_scale: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None):
    """Chunkwise forward.  Returns (o [B,T,Hv,dv], ht [B,Hv,dk,dv] or None).
    ``out_f32`` writes o in fp32 (the unrounded accumulator) instead of the input dtype.
    ``bwd_cache``: a device byte tensor of gdn_chunk_fwd_cache_size() bytes that the forward fills
    for gdn_chunk_bwd(..., fwd_cache=) over the same inputs."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    if o is None:
        o = torch.empty((B, T, Hv, dv), dtype=torch.float32 if out_f32 else q.dtype, device=q.device)
    if ht is None and want_ht:
        ht = torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=q.device)
    lib = load()
    a, keep = fwd_args(q, k, v, alpha, b, w, beta, h0, z, head_map, scale, o, ht, bwd_cache, alpha_scale)
    need = lib.gdn_chunk_fwd_workspace_size(ctypes.byref(a))
    ws = _workspace(need, q.device, workspace)
    check(lib.gdn_chunk_fwd(ctypes.byref(a), _ptr(ws), need, _stream(stream)), "gdn_chunk_fwd")
    return o, ht


def gdn_chunk_fwd_noalloc(q, k, v, alpha, b=None, w=None, beta=None, h0=None, z=None, head_map=None,
                          scale: float = 1.0, *, o=None, ht=None, want_ht: bool = True, out_f32: bool = False,
                          stream=None):
    """gdn_chunk_fwd with the library's built-in 16 MiB scratch instead of a workspace (calls on one
    device must not overlap in time).  Returns (o, ht)."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    if o is None:
        o = torch.empty((B, T, Hv, dv), dtype=torch.float32 if out_f32 else q.dtype, device=q.device)
    if ht is None and want_ht:
        ht = torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=q.device)
    lib = load()
    a, keep = fwd_args(q, k, v, alpha, b, w, beta, h0, z, head_map, scale, o, ht)
    check(lib.gdn_chunk_fwd_noalloc(ctypes.byref(a), _stream(stream)), "gdn_chunk_fwd_noalloc")
    return o, ht


def gdn_chunk_fwd_noalloc_status(stream=None) -> int:
    """The status word of the built-in scratch after gdn_chunk_fwd_noalloc calls (synchronises
    ``stream``): 0, or GDN_ERR_TIMEOUT (5) if a bounded wait inside a kernel expired."""
    return int(load().gdn_chunk_fwd_noalloc_status(_stream(stream)))


def gdn_segment_map(q, k, v, alpha, b=None, w=None, beta=None, head_map=None, *, want_o: bool = False,
                    workspace: Optional[torch.Tensor] = None, stream=None):
    """The affine map of this segment of every sequence on the state: returns (M [B,Hv,dk,dk],
    N [B,Hv,dk,dv]) with state_after = M state_before + N, plus the segment's output from a zero
    entering state when ``want_o`` (then (M, N, o))."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    M = torch.empty((B, Hv, dk, dk), dtype=torch.float32, device=q.device)
    N = torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=q.device)
    o = torch.empty((B, T, Hv, dv), dtype=q.dtype, device=q.device) if want_o else None
    lib = load()
    a, keep = fwd_args(q, k, v, alpha, b, w, beta, None, None, head_map, 1.0, o, N)
    need = lib.gdn_segment_map_workspace_size(ctypes.byref(a))
    ws = _workspace(need, q.device, workspace)
    check(lib.gdn_segment_map(ctypes.byref(a), _ptr(M), _ptr(ws), need, _stream(stream)), "gdn_segment_map")
    return (M, N, o) if want_o else (M, N)


def gdn_state_compose(M, N, S, *, transpose: bool = False, out: Optional[torch.Tensor] = None, stream=None):
    """op(M) S + N per (sequence, head) on the device, op = transpose or identity.  M [..., dk, dk],
    N and S [..., dk, dv] fp32 (S or N may be None: zero).  Returns the result (``out`` if given)."""
    ref = S if S is not None else N
    dk, dv = M.shape[-1], ref.shape[-1]
    pairs = M.numel() // (dk * dk)
    if out is None:
        out = torch.empty(ref.shape, dtype=torch.float32, device=M.device)
    check(load().gdn_state_compose(_ptr(M), _ptr(N), _ptr(S), _ptr(out), pairs, dk, dv, int(transpose),
                                   _stream(stream)), "gdn_state_compose")
    return out


def bwd_args(q, k, v, alpha, b=None, w=None, beta=None, h0=None, head_map=None, scale=1.0,
             grad_o=None, grad_ht=None, grads=None, fwd_cache=None, alpha_scale=None,
             grads_in_dtype: bool = False) -> Tuple[BwdArgs, list]:
    bb, ww, gpc = _gates(alpha, b, w, beta)
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    hm = _head_map(head_map, q.device, q.shape[-2])
    g = grads
    tp, ts = _inputs(2, q, k, v, alpha, bb, ww)
    a = BwdArgs(q=tp["q"], k=tp["k"], v=tp["v"], alpha=tp["alpha"], b=tp["b"], w=tp["w"],
                h0=_ptr(h0), head_map=_ptr(hm), grad_o=_ptr(grad_o), grad_ht=_ptr(grad_ht),
                grad_q=_ptr(g["dq"]), grad_k=_ptr(g["dk"]), grad_v=_ptr(g["dv"]),
                grad_alpha=_ptr(g["dalpha"]), grad_b=_ptr(g["db"] if gpc else g["dbeta"]),
                grad_w=_ptr(g.get("dw")), grad_h0=_ptr(g.get("dh0")),
                B=B, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv, scale=scale,
                alpha_per_channel=int(alpha.dim() == 4), gates_per_channel=gpc,
                dtype=_dt(q), gate_dtype=_dt(alpha), fwd_cache=_ptr(fwd_cache),
                fwd_cache_bytes=0 if fwd_cache is None else fwd_cache.numel() * fwd_cache.element_size(),
                gate_logits=int(alpha_scale is not None), alpha_scale=_ptr(alpha_scale),
                grad_alpha_scale=_ptr(g.get("dalpha_scale")), grads_in_dtype=int(grads_in_dtype), strides=ts)
    return a, [q, k, v, alpha, bb, ww, h0, hm, grad_o, grad_ht, g, fwd_cache, alpha_scale]


def gdn_chunk_bwd(q, k, v, alpha, b=None, w=None, beta=None, h0=None, head_map=None,
                  scale: float = 1.0, *, grad_o, grad_ht=None, want_dh0: bool = True,
                  fwd_cache: Optional[torch.Tensor] = None, alpha_scale: Optional[torch.Tensor] = None,
                  grads_in_dtype: bool = False, workspace: Optional[torch.Tensor] = None,
                  stream=None) -> Dict[str, torch.Tensor]:
    """Chunkwise backward.  Returns dq, dk, dv, dalpha and db/dw (or dbeta) in fp32, or with
    ``grads_in_dtype`` in the dtypes of q and of the gates; dh0 in fp32.
    ``fwd_cache``: the cache a gdn_chunk_fwd(..., bwd_cache=) call filled with these same inputs
    (the forward is then not recomputed).  With ``alpha_scale`` the gates are logits: dalpha, db,
    dw, dbeta are the gradients of the logits, and dalpha_scale [Hv] that of alpha_scale."""
    bb, ww, gpc = _gates(alpha, b, w, beta)
    like = lambda t: torch.empty(t.shape, dtype=t.dtype if grads_in_dtype else torch.float32, device=t.device)
    grads = {"dq": like(q), "dk": like(k), "dv": like(v), "dalpha": like(alpha)}
    if gpc:
        grads["db"] = like(b)
        grads["dw"] = like(w)
    else:
        grads["dbeta"] = like(beta)
    if want_dh0:
        B, T, Hk, dk = q.shape
        Hv, dv = v.shape[2], v.shape[3]
        grads["dh0"] = torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=q.device)
    if alpha_scale is not None:
        grads["dalpha_scale"] = torch.empty(tuple(alpha_scale.shape), dtype=torch.float32, device=q.device)
    lib = load()
    a, keep = bwd_args(q, k, v, alpha, b, w, beta, h0, head_map, scale, grad_o, grad_ht, grads, fwd_cache,
                       alpha_scale, grads_in_dtype)
    need = lib.gdn_chunk_bwd_workspace_size(ctypes.byref(a))
    ws = _workspace(need, q.device, workspace)
    check(lib.gdn_chunk_bwd(ctypes.byref(a), _ptr(ws), need, _stream(stream)), "gdn_chunk_bwd")
    return grads


def gdn_decode_step(state, q, k, v, alpha, b=None, w=None, beta=None, head_map=None,
                    scale: float = 1.0, *, conv_state=None, conv_w=None, z=None, o=None,
                    out_f32: bool = False, alpha_scale=None, stream=None):
    """One token for N sequences; ``state`` [N,Hv,dk,dv] fp32 is updated in place.  Returns o."""
    bb, ww, gpc = _gates(alpha, b, w, beta)
    N, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if o is None:
        o = torch.empty((N, Hv, dv), dtype=torch.float32 if out_f32 else q.dtype, device=q.device)
    hm = _head_map(head_map, q.device, q.shape[-2])
    tp, ts = _inputs(1, q, k, v, alpha, bb, ww, z)
    a = DecodeArgs(q=tp["q"], k=tp["k"], v=tp["v"], alpha=tp["alpha"], b=tp["b"], w=tp["w"],
                   state=_ptr(state), o=_ptr(o), head_map=_ptr(hm), conv_state=_ptr(conv_state),
                   conv_w=_ptr(conv_w), z=tp["z"], N=N, Hk=Hk, Hv=Hv, dk=dk, dv=dv, scale=scale,
                   alpha_per_channel=int(alpha.dim() == 3), gates_per_channel=gpc,
                   dtype=_dt(q), gate_dtype=_dt(alpha),
                   out_f32=int(o.dtype == torch.float32 and q.dtype != torch.float32),
                   gate_logits=int(alpha_scale is not None), alpha_scale=_ptr(alpha_scale), strides=ts)
    check(load().gdn_decode_step(ctypes.byref(a), _stream(stream)), "gdn_decode_step")
    return o


NORM_EPS = 1e-6  # the output norm's epsilon when the caller gives none


def _layer_args(xq, xk, xv, conv_w, alpha, z, b, w, beta, h0, head_map, scale, y=None, ht=None, cs=None,
                out_f32=0, bwd_cache=None, norm_w=None, norm_eps=NORM_EPS, alpha_scale=None):
    bb, ww, gpc = _gates(alpha, b, w, beta)
    B, T, Hk, dk = xq.shape
    Hv, dv = xv.shape[2], xv.shape[3]
    hm = _head_map(head_map, xq.device, xq.shape[-2])
    tp, ts = _inputs(2, xq, xk, xv, alpha, bb, ww, z)
    a = LayerArgs(xq=tp["q"], xk=tp["k"], xv=tp["v"], conv_w=_ptr(conv_w), alpha=tp["alpha"],
                  b=tp["b"], w=tp["w"], z=tp["z"], h0=_ptr(h0), y=_ptr(y), ht=_ptr(ht),
                  conv_state_out=_ptr(cs), head_map=_ptr(hm), B=B, T=T, Hk=Hk, Hv=Hv, dk=dk,
                  dv=dv, scale=scale, alpha_per_channel=int(alpha.dim() == 4),
                  gates_per_channel=gpc, dtype=_dt(xq), gate_dtype=_dt(alpha), out_f32=out_f32,
                  bwd_cache=_ptr(bwd_cache), bwd_cache_bytes=bwd_cache.numel() if bwd_cache is not None else 0,
                  norm_w=_ptr(norm_w), norm_eps=norm_eps, gate_logits=int(alpha_scale is not None),
                  alpha_scale=_ptr(alpha_scale), strides=ts)
    return a, hm


def gdn_layer_core_fwd_cache_size(xq, xk, xv, conv_w, alpha, z, b=None, w=None, beta=None, h0=None,
                                  head_map=None, scale: float = 1.0, norm_w=None) -> int:
    """Bytes of the layer forward's optional backward cache (0 where it cannot keep one)."""
    a, _ = _layer_args(xq, xk, xv, conv_w, alpha, z, b, w, beta, h0, head_map, scale, norm_w=norm_w)
    return int(load().gdn_layer_core_fwd_cache_size(ctypes.byref(a)))


def gdn_layer_core_fwd(xq, xk, xv, conv_w, alpha, z, b=None, w=None, beta=None, h0=None,
                       head_map=None, scale: float = 1.0, *, want_ht: bool = True,
                       want_conv_state: bool = False, y=None, out_f32: bool = False,
                       bwd_cache: Optional[torch.Tensor] = None, norm_w=None, norm_eps: float = NORM_EPS,
                       alpha_scale=None, workspace: Optional[torch.Tensor] = None, stream=None):
    """GQA layer core forward.  Returns (y, ht or None, conv_state or None).  ``bwd_cache``: a
    uint8 device tensor of gdn_layer_core_fwd_cache_size() bytes that a later
    gdn_layer_core_bwd(..., fwd_cache=) over the same inputs reads.  ``norm_w`` [dv] (the layer's
    dtype): the output norm before the gate, y = RMSNorm(o) * norm_w * swish(z)."""
    B, T, Hk, dk = xq.shape
    Hv, dv = xv.shape[2], xv.shape[3]
    if y is None:
        y = torch.empty((B, T, Hv, dv), dtype=torch.float32 if out_f32 else xq.dtype, device=xq.device)
    ht = torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=xq.device) if want_ht else None
    cs = (torch.empty((B, 2 * Hk * dk + Hv * dv, 3), dtype=xq.dtype, device=xq.device)
          if want_conv_state else None)
    a, hm = _layer_args(xq, xk, xv, conv_w, alpha, z, b, w, beta, h0, head_map, scale, y=y, ht=ht, cs=cs,
                        out_f32=int(y.dtype == torch.float32 and xq.dtype != torch.float32), bwd_cache=bwd_cache,
                        norm_w=norm_w, norm_eps=norm_eps, alpha_scale=alpha_scale)
    lib = load()
    need = lib.gdn_layer_core_fwd_workspace_size(ctypes.byref(a))
    ws = _workspace(need, xq.device, workspace)
    check(lib.gdn_layer_core_fwd(ctypes.byref(a), _ptr(ws), need, _stream(stream)),
          "gdn_layer_core_fwd")
    return y, ht, cs


def gdn_layer_core_bwd(xq, xk, xv, conv_w, alpha, z, grad_y, b=None, w=None, beta=None, h0=None,
                       grad_ht=None, head_map=None, scale: float = 1.0, *, want_h0_grad: bool = True,
                       fwd_cache: Optional[torch.Tensor] = None, norm_w=None, norm_eps: float = NORM_EPS,
                       alpha_scale=None, workspace: Optional[torch.Tensor] = None,
                       stream=None) -> Dict[str, torch.Tensor]:
    """GQA layer core backward (reverse mode of gdn_layer_core_fwd).  Returns a dict of fp32
    gradients: dxq, dxk, dxv, dconv_w, dalpha, dz, dh0 (or None), db/dw or dbeta, and dnorm_w
    with the output norm (``norm_w``).
    ``fwd_cache``: the cache a gdn_layer_core_fwd(..., bwd_cache=) call filled with these inputs."""
    bb, ww, gpc = _gates(alpha, b, w, beta)
    B, T, Hk, dk = xq.shape
    Hv, dv = xv.shape[2], xv.shape[3]
    dev = xq.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dxq": torch.empty((B, T, Hk, dk), **f32), "dxk": torch.empty((B, T, Hk, dk), **f32),
           "dxv": torch.empty((B, T, Hv, dv), **f32), "dconv_w": torch.empty(tuple(conv_w.shape), **f32),
           "dalpha": torch.empty(tuple(alpha.shape), **f32), "dz": torch.empty((B, T, Hv, dv), **f32),
           "dh0": torch.empty((B, Hv, dk, dv), **f32) if want_h0_grad else None}
    if gpc:
        out["db"] = torch.empty(tuple(bb.shape), **f32)
        out["dw"] = torch.empty(tuple(ww.shape), **f32)
        gb, gw = out["db"], out["dw"]
    else:
        out["dbeta"] = torch.empty(tuple(bb.shape), **f32)
        gb, gw = out["dbeta"], None
    if norm_w is not None:
        out["dnorm_w"] = torch.empty((dv,), **f32)
    if alpha_scale is not None:
        out["dalpha_scale"] = torch.empty(tuple(alpha_scale.shape), **f32)
    hm = _head_map(head_map, dev, Hk)
    tp, ts = _inputs(2, xq, xk, xv, alpha, bb, ww, z)
    a = LayerBwdArgs(xq=tp["q"], xk=tp["k"], xv=tp["v"], conv_w=_ptr(conv_w), alpha=tp["alpha"],
                     b=tp["b"], w=tp["w"], z=tp["z"], h0=_ptr(h0), head_map=_ptr(hm), grad_y=_ptr(grad_y),
                     grad_ht=_ptr(grad_ht), grad_xq=_ptr(out["dxq"]), grad_xk=_ptr(out["dxk"]),
                     grad_xv=_ptr(out["dxv"]), grad_conv_w=_ptr(out["dconv_w"]), grad_alpha=_ptr(out["dalpha"]),
                     grad_b=_ptr(gb), grad_w=_ptr(gw), grad_z=_ptr(out["dz"]), grad_h0=_ptr(out["dh0"]),
                     B=B, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv, scale=scale,
                     alpha_per_channel=int(alpha.dim() == 4), gates_per_channel=gpc, dtype=_dt(xq),
                     gate_dtype=_dt(alpha), fwd_cache=_ptr(fwd_cache),
                     fwd_cache_bytes=fwd_cache.numel() if fwd_cache is not None else 0,
                     norm_w=_ptr(norm_w), norm_eps=norm_eps, grad_norm_w=_ptr(out.get("dnorm_w")),
                     gate_logits=int(alpha_scale is not None), alpha_scale=_ptr(alpha_scale),
                     grad_alpha_scale=_ptr(out.get("dalpha_scale")), strides=ts)
    lib = load()
    need = lib.gdn_layer_core_bwd_workspace_size(ctypes.byref(a))
    ws = _workspace(need, dev, workspace)
    check(lib.gdn_layer_core_bwd(ctypes.byref(a), _ptr(ws), need, _stream(stream)), "gdn_layer_core_bwd")
    return out
