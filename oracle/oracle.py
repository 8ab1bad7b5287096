"""TEST INFRASTRUCTURE ONLY: numpy front end of the fp64 CPU oracle (gdn_oracle.cpp).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference leg may import
this module.  The product path (the CUDA library and its Python binding) never does.

All functions take numpy arrays or torch CPU tensors (any float dtype; bf16 is upcast exactly)
in the token-major layouts of the library and return float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with plain g++ (-O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _LIB + ".tmp"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def load_library(path: str):
    """Bind the oracle's C entry points from a compiled library at ``path``."""
    lib = ctypes.CDLL(path)
    _declare(lib)
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = load_library(_LIB)
    return _lib


def _declare(lib):
    if True:
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        common = [P] * 8 + [I] * 9 + [D]
        lib.oracle_fwd.argtypes = common + [P, I, P, P, I]
        lib.oracle_bwd.argtypes = common + [P, P, P, I] + [P] * 7 + [I]
        lib.oracle_chunk_fwd.argtypes = common + [I, P, P, I]
        lib.oracle_conv_silu.argtypes = [P, P, P, I, I, I, P, P]
        lib.oracle_l2norm_rows.argtypes = [P, ctypes.c_long, I, D]
        lib.oracle_l2norm_rows.restype = None
        lib.oracle_swish_gate.argtypes = [P, P, ctypes.c_long, P]
        lib.oracle_swish_gate.restype = None
        for f in (lib.oracle_fwd, lib.oracle_bwd, lib.oracle_chunk_fwd, lib.oracle_conv_silu):
            f.restype = ctypes.c_int


def threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def f64(x) -> Optional[np.ndarray]:
    """Exact upcast to a contiguous float64 array (torch bf16/f32 tensors or numpy)."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class _Args:
    """Normalised recurrence inputs.  Scalar beta is passed as both b and w."""

    def __init__(self, q, k, v, alpha, b=None, w=None, beta=None, h0=None, head_map=None,
                 scale: float = 1.0):
        self.q, self.k, self.v = f64(q), f64(k), f64(v)
        B, T, Hk, dk = self.q.shape
        Hv, dv = self.v.shape[2], self.v.shape[3]
        self.dims = (B, T, Hk, Hv, dk, dv)
        a = f64(alpha)
        self.a_ch = 1 if a.ndim == 3 else a.shape[3]
        self.alpha = a.reshape(B, T, Hv, self.a_ch)
        if beta is not None:
            bb = f64(beta).reshape(B, T, Hv, 1)
            self.bg, self.wg = bb, bb
            self.scalar_beta = True
        else:
            bg, wg = f64(b), f64(w)
            self.bg = bg if bg.ndim == 4 else bg.reshape(B, T, Hv, 1)
            self.wg = wg if wg.ndim == 4 else wg.reshape(B, T, Hv, 1)
            self.scalar_beta = False
        self.b_ch, self.w_ch = self.bg.shape[3], self.wg.shape[3]
        self.h0 = f64(h0)
        if head_map is None:
            head_map = np.arange(Hv) // (Hv // Hk)
        self.map = np.ascontiguousarray(np.asarray(head_map, dtype=np.int32))
        self.scale = float(scale)

    def common(self):
        B, T, Hk, Hv, dk, dv = self.dims
        return [_ptr(self.q), _ptr(self.k), _ptr(self.v), _ptr(self.alpha), _ptr(self.bg),
                _ptr(self.wg), _ptr(self.h0), _ptr(self.map), B, T, Hk, Hv, dk, dv,
                self.a_ch, self.b_ch, self.w_ch, self.scale]


def _pairs(pairs: Optional[Sequence[int]]):
    if pairs is None:
        return None, 0, None
    arr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32))
    return _ptr(arr), len(arr), arr


def fwd(q, k, v, alpha, b=None, w=None, beta=None, h0=None, head_map=None, scale=1.0,
        pairs: Optional[Sequence[int]] = None, nthreads: Optional[int] = None):
    """Sequential recurrence.  Returns (o [B,T,Hv,dv], hT [B,Hv,dk,dv]).

    ``pairs`` restricts the work to flattened (b * Hv + hv) indices; other entries are NaN."""
    a = _Args(q, k, v, alpha, b, w, beta, h0, head_map, scale)
    B, T, Hk, Hv, dk, dv = a.dims
    o = np.full((B, T, Hv, dv), np.nan)
    hT = np.full((B, Hv, dk, dv), np.nan)
    pp, npairs, keep = _pairs(pairs)
    rc = _load().oracle_fwd(*a.common(), pp, npairs, _ptr(o), _ptr(hT), nthreads or threads())
    if rc:
        raise ValueError("oracle_fwd: inconsistent sizes")
    return o, hT


def bwd(q, k, v, alpha, b=None, w=None, beta=None, h0=None, head_map=None, scale=1.0,
        dout=None, dht=None, pairs: Optional[Sequence[int]] = None,
        nthreads: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Reverse mode of fwd().  Returns dq, dk [B,T,Hk,dk] (summed over the value heads of each
    key head, ascending), dv, dalpha, db/dw or dbeta, dh0, plus dq_v/dk_v per value head."""
    a = _Args(q, k, v, alpha, b, w, beta, h0, head_map, scale)
    B, T, Hk, Hv, dk, dv = a.dims
    go = f64(dout)
    gh = f64(dht)
    nan = np.nan
    dq_v = np.full((B, T, Hv, dk), nan)
    dk_v = np.full((B, T, Hv, dk), nan)
    dv_ = np.full((B, T, Hv, dv), nan)
    da = np.full((B, T, Hv, a.a_ch), nan)
    db = np.full((B, T, Hv, a.b_ch), nan)
    dw = np.full((B, T, Hv, a.w_ch), nan)
    dh0 = np.full((B, Hv, dk, dv), nan)
    pp, npairs, keep = _pairs(pairs)
    rc = _load().oracle_bwd(*a.common(), _ptr(go), _ptr(gh), pp, npairs, _ptr(dq_v), _ptr(dk_v),
                            _ptr(dv_), _ptr(da), _ptr(db), _ptr(dw), _ptr(dh0),
                            nthreads or threads())
    if rc:
        raise ValueError("oracle_bwd: inconsistent sizes")
    dq = np.zeros((B, T, Hk, dk))
    dkk = np.zeros((B, T, Hk, dk))
    for hv in range(Hv):
        dq[:, :, a.map[hv]] += dq_v[:, :, hv]
        dkk[:, :, a.map[hv]] += dk_v[:, :, hv]
    out = {"dq": dq, "dk": dkk, "dv": dv_, "dh0": dh0, "dq_v": dq_v, "dk_v": dk_v}
    out["dalpha"] = da if alpha_is_channel(a) else da[..., 0]
    if a.scalar_beta:
        out["dbeta"] = db[..., 0] + dw[..., 0]
    else:
        out["db"] = db if a.b_ch > 1 else db[..., 0]
        out["dw"] = dw if a.w_ch > 1 else dw[..., 0]
    return out


def alpha_is_channel(a: _Args) -> bool:
    return a.a_ch > 1


def chunk_fwd(q, k, v, alpha, b=None, w=None, beta=None, h0=None, head_map=None, scale=1.0,
              C: int = 64, nthreads: Optional[int] = None):
    """The chunkwise (WY) form written out plainly.  Returns (o, hT)."""
    a = _Args(q, k, v, alpha, b, w, beta, h0, head_map, scale)
    B, T, Hk, Hv, dk, dv = a.dims
    o = np.full((B, T, Hv, dv), np.nan)
    hT = np.full((B, Hv, dk, dv), np.nan)
    rc = _load().oracle_chunk_fwd(*a.common(), int(C), _ptr(o), _ptr(hT), nthreads or threads())
    if rc:
        raise ValueError("oracle_chunk_fwd: inconsistent sizes")
    return o, hT


# ---- gates from logits -----------------------------------------------------------------------
# The gates as functions of the layer's projections (explainer «Architecture et versions hybrides»,
# Figure 1 caption: alpha takes the Mamba-2 parametrisation; zubnet.ai news item: the erase and write
# gates are two sigmoids): alpha = exp(-a_h softplus(x)) with a positive scale a_h per value head (the
# Mamba-2 form exp(-A dt), dt = softplus(x), A = a_h), and b, w, beta = sigmoid(x).

def _softplus(x):
    return np.logaddexp(0.0, x)


def gates_from_logits(x_alpha, a_scale, x_b=None, x_w=None, x_beta=None):
    """(alpha, b, w, beta) from their logits; a_scale [Hv] (alpha's last axis is the channel axis when
    it has one, the value head is axis 2)."""
    xa = f64(x_alpha)
    a = f64(a_scale)
    ah = a.reshape((1, 1, -1) + (1,) * (xa.ndim - 3))
    alpha = np.exp(-ah * _softplus(xa))
    sig = lambda x: None if x is None else _sigmoid(f64(x))
    return alpha, sig(x_b), sig(x_w), sig(x_beta)


def logit_grads(x_alpha, a_scale, dalpha, x_b=None, db=None, x_w=None, dw=None, x_beta=None, dbeta=None):
    """Chain rule from the gradients of the gates to those of their logits and of a_h:
        d x_alpha = dalpha * alpha * (-a_h sigmoid(x)),   d a_h = sum dalpha * alpha * (-softplus(x)),
        d x = dg * g (1 - g) for the sigmoid gates."""
    xa, a = f64(x_alpha), f64(a_scale)
    ah = a.reshape((1, 1, -1) + (1,) * (xa.ndim - 3))
    alpha = np.exp(-ah * _softplus(xa))
    out = {"dalpha": f64(dalpha) * alpha * (-ah * _sigmoid(xa))}
    axes = (0, 1) + tuple(range(3, xa.ndim))
    out["dalpha_scale"] = np.sum(f64(dalpha) * alpha * (-_softplus(xa)), axis=axes)
    for name, x, d in (("db", x_b, db), ("dw", x_w, dw), ("dbeta", x_beta, dbeta)):
        if x is not None:
            g = _sigmoid(f64(x))
            out[name] = f64(d) * g * (1.0 - g)
    return out


def segment_map(q, k, v, alpha, b=None, w=None, beta=None, head_map=None):
    """The affine map by which one segment of a sequence acts on the state.

    For the state S_in entering the segment, the state after it is M S_in + N (per (batch, value
    head)), because each token's update is affine in the state (GDN-2 summary, «Méthodologie» §1):
        S_t = A_t S_{t-1} + k_t z_t^T,   A_t = (I - k_t e_t^T) Diag(alpha_t),  e = b .* k,  z = w .* v
    so M = A_T ... A_1 (dk x dk, the transitions multiplied out here one token at a time) and N is
    the state after the segment entered with zeros (fwd() from a zero state).
    Returns (M [B,Hv,dk,dk], N [B,Hv,dk,dv])."""
    a = _Args(q, k, v, alpha, b, w, beta, None, head_map, 1.0)
    B, T, Hk, Hv, dk, dv = a.dims
    M = np.empty((B, Hv, dk, dk))
    for bb in range(B):
        for hv in range(Hv):
            hk = a.map[hv]
            m = np.eye(dk)
            for t in range(T):
                kk = a.k[bb, t, hk]
                al = np.broadcast_to(a.alpha[bb, t, hv], (dk,))
                e = np.broadcast_to(a.bg[bb, t, hv], (dk,)) * kk
                m = al[:, None] * m                # Diag(alpha_t) M
                m = m - np.outer(kk, e @ m)       # (I - k e^T) Diag(alpha_t) M
            M[bb, hv] = m
    _, N = fwd(q, k, v, alpha, b=b, w=w, beta=beta, head_map=head_map)
    return M, N


def compose(M, N, S, transpose: bool = False):
    """M S + N (or M^T S + N) for every (batch, head): the state after a segment given the state
    entering it, or, transposed, a state gradient carried back across a segment."""
    M, N, S = f64(M), f64(N), f64(S)
    Mt = np.swapaxes(M, -1, -2) if transpose else M
    return np.einsum("bhij,bhjk->bhik", Mt, S) + N


def decode_step(state, q, k, v, alpha, b=None, w=None, beta=None, head_map=None, scale=1.0,
                pairs: Optional[Sequence[int]] = None):
    """One token for N sequences: q,k [N,Hk,dk], v [N,Hv,dv], gates [N,Hv,(d)], state
    [N,Hv,dk,dv].  Returns (o [N,Hv,dv], new state)."""
    def tok1(x):
        x = f64(x)
        return None if x is None else x[:, None]
    o, hT = fwd(tok1(q), tok1(k), tok1(v), tok1(alpha), tok1(b), tok1(w), tok1(beta),
                h0=state, head_map=head_map, scale=scale, pairs=pairs)
    return o[:, 0], hT


def conv_silu(x, conv_w, hist=None):
    """Causal depthwise conv (kernel 4, no bias) + SiLU over x [B,T,Cch].
    Returns (y [B,T,Cch], last three inputs [B,Cch,3])."""
    x = f64(x)
    B, T, Cch = x.shape
    w = f64(conv_w)
    h = f64(hist)
    y = np.empty_like(x)
    hist_out = np.empty((B, Cch, 3))
    rc = _load().oracle_conv_silu(_ptr(x), _ptr(w), _ptr(h), B, T, Cch, _ptr(y), _ptr(hist_out))
    if rc:
        raise ValueError("oracle_conv_silu: bad sizes")
    return y, hist_out


L2_EPS = 1e-6


def l2norm(x, eps: float = L2_EPS):
    x = f64(x).copy()
    _load().oracle_l2norm_rows(_ptr(x), x.size // x.shape[-1], x.shape[-1], float(eps))
    return x


RMS_EPS = 1e-6


def gated_rmsnorm(o, z, norm_w, eps: float = RMS_EPS):
    """The layer's output norm and gate (explainer «Architecture et versions hybrides», Figure 1
    caption: the output is normalised, then multiplied by a gate; mkdocs chapter «Gated DeltaNet»,
    «Le décompte»: 128 norm weights shared by the heads): every (token, head) row of dv values is
    divided by its root mean square, scaled by norm_w [dv], and multiplied by z sigmoid(z)."""
    o, z, wn = f64(o), f64(z), f64(norm_w)
    r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return o * r * wn * z * _sigmoid(z)


def swish_gate(o, z):
    o = f64(o)
    z = f64(z)
    y = np.empty_like(o)
    _load().oracle_swish_gate(_ptr(o), _ptr(z), o.size, _ptr(y))
    return y


def layer_core_fwd(xq, xk, xv, conv_w, alpha, beta, z, head_map=None, scale=1.0, h0=None,
                   pairs: Optional[Sequence[int]] = None, norm_w=None):
    """GQA layer core: conv(k=4)+SiLU on the q, k, v projections (zero history), L2 norm on
    q and k, the recurrence, then the swish(z) output gate.  Conv channels are ordered
    q (Hk*dk), k (Hk*dk), v (Hv*dv).  Returns (y [B,T,Hv,dv], hT)."""
    xq, xk, xv = f64(xq), f64(xk), f64(xv)
    w = f64(conv_w)
    B, T, Hk, dk = xq.shape
    Hv, dv = xv.shape[2], xv.shape[3]
    cq = Hk * dk
    q, _ = conv_silu(xq.reshape(B, T, cq), w[:cq])
    k, _ = conv_silu(xk.reshape(B, T, cq), w[cq:2 * cq])
    v, _ = conv_silu(xv.reshape(B, T, Hv * dv), w[2 * cq:])
    q = l2norm(q.reshape(B, T, Hk, dk))
    k = l2norm(k.reshape(B, T, Hk, dk))
    v = v.reshape(B, T, Hv, dv)
    o, hT = fwd(q, k, v, alpha, beta=beta, h0=h0, head_map=head_map, scale=scale, pairs=pairs)
    if norm_w is not None:
        return gated_rmsnorm(o, z, norm_w), hT
    return swish_gate(o, z), hT


# ---- layer-core backward (reverse mode of layer_core_fwd, fp64 numpy) ---------------------------
# The layer of the explainer's «Architecture et versions hybrides» (Figure 1 caption) and the mkdocs
# chapter «Gated DeltaNet»: per channel a causal depthwise convolution of kernel 4 (zero history,
# conv_w[ch][3] weighting the current token), SiLU, then the L2 norm of each q and k head row; the
# recurrence; the swish(z) output gate.  Each reverse step below is the derivative of one forward
# step, written out; the finite-difference pin in tests/ checks the composition.

def _conv_pre(x, w):
    """Causal depthwise conv, kernel 4, zero history: u[:, t, c] = sum_tap w[c, tap] x[:, t-3+tap, c]."""
    B, T, C = x.shape
    u = np.zeros_like(x)
    for tap in range(4):
        sh = 3 - tap
        if sh == 0:
            u += w[:, tap] * x
        elif sh < T:
            u[:, sh:] += w[:, tap] * x[:, :T - sh]
    return u


def _conv_pre_bwd(x, w, du):
    """Reverse of _conv_pre: dx[:, s] = sum_tap w[tap] du[:, s+3-tap]; dw[c, tap] = sum du[t] x[t-3+tap]."""
    B, T, C = x.shape
    dx = np.zeros_like(x)
    dw = np.zeros((C, 4))
    for tap in range(4):
        sh = 3 - tap
        if sh == 0:
            dx += w[:, tap] * du
            dw[:, tap] = np.sum(du * x, axis=(0, 1))
        elif sh < T:
            dx[:, :T - sh] += w[:, tap] * du[:, sh:]
            dw[:, tap] = np.sum(du[:, sh:] * x[:, :T - sh], axis=(0, 1))
    return dx, dw


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def layer_core_bwd(xq, xk, xv, conv_w, alpha, z, dy, b=None, w=None, beta=None, head_map=None,
                   scale=1.0, h0=None, dht=None, norm_w=None) -> Dict[str, np.ndarray]:
    """Reverse mode of the GQA layer core for loss gradients dy (of y) and dht (of the final
    state).  Returns dxq, dxk, dxv, dconv_w, dz, dalpha, db/dw or dbeta, dh0, and dnorm_w when the
    output norm is on (norm_w given)."""
    xq, xk, xv, W = f64(xq), f64(xk), f64(xv), f64(conv_w)
    zz, g = f64(z), f64(dy)
    B, T, Hk, dk = xq.shape
    Hv, dv = xv.shape[2], xv.shape[3]
    cq = Hk * dk
    parts = {}
    for name, x, wsl, H, d, norm in (("q", xq, W[:cq], Hk, dk, True), ("k", xk, W[cq:2 * cq], Hk, dk, True),
                                     ("v", xv, W[2 * cq:], Hv, dv, False)):
        xf = x.reshape(B, T, H * d)
        u = _conv_pre(xf, wsl)
        a = u * _sigmoid(u)                          # SiLU
        if norm:
            a4 = a.reshape(B, T, H, d)
            n = np.sqrt(np.sum(a4 * a4, axis=-1, keepdims=True) + L2_EPS)
            out = a4 / n                             # L2 norm of each head row
        else:
            n, out = None, a.reshape(B, T, H, d)
        parts[name] = (xf, wsl, u, a, n, out)
    q, k, v = parts["q"][5], parts["k"][5], parts["v"][5]
    gk = dict(beta=beta) if beta is not None else dict(b=b, w=w)
    o, _ = fwd(q, k, v, alpha, head_map=head_map, scale=scale, h0=h0, **gk)
    sg = _sigmoid(zz)
    swz = zz * sg                                    # swish(z)
    dswz = sg + zz * sg * (1.0 - sg)                 # its derivative
    extra = {}
    if norm_w is None:
        do = g * swz                                 # y = o * swish(z)
        dz = g * o * dswz
    else:
        # y = n * wn * swish(z),  n = o * r,  r = (mean_j o_j^2 + eps)^(-1/2) per (token, head) row
        wn = f64(norm_w)
        r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + RMS_EPS)
        n = o * r
        dn = g * wn * swz
        dz = g * n * wn * dswz
        extra["dnorm_w"] = np.sum(g * n * swz, axis=(0, 1, 2))
        do = r * (dn - n * np.mean(dn * n, axis=-1, keepdims=True))
    core = bwd(q, k, v, alpha, head_map=head_map, scale=scale, h0=h0, dout=do, dht=dht, **gk)
    res = {"dz": dz, "dalpha": core["dalpha"], "dh0": core["dh0"], **extra}
    for key in ("dbeta", "db", "dw"):
        if key in core:
            res[key] = core[key]
    dconv = []
    for name, gout in (("q", core["dq"]), ("k", core["dk"]), ("v", core["dv"])):
        xf, wsl, u, a, n, out = parts[name]
        if n is not None:                            # out = a / n,  n = sqrt(sum a^2 + eps)
            dot = np.sum(out * gout, axis=-1, keepdims=True)
            da = ((gout - out * dot) / n).reshape(a.shape)
        else:
            da = gout.reshape(a.shape)
        s = _sigmoid(u)
        du = da * (s + u * s * (1.0 - s))            # d/du of u * sigmoid(u)
        dx, dwc = _conv_pre_bwd(xf, wsl, du)
        res["dx" + name] = dx.reshape(parts[name][5].shape)
        dconv.append(dwc)
    res["dconv_w"] = np.concatenate(dconv, axis=0)
    return res
