"""Seeded synthetic inputs for the gated delta-rule workloads.

This module is shared by the tests, the benchmark and the CPU oracle's callers.  It holds
none of the recurrence's arithmetic: it draws random numbers, applies the input recipe
(L2-normalised q/k rows, squashed gates), and casts once to the stated dtype.  Everything
it returns lives on the host (torch CPU tensors); callers move it where they need it.

Recipe (one numpy ``default_rng`` stream per workload, draws in this fixed order):
  q, k, v, alpha-logits, b-logits (or beta-logits), w-logits, [z, conv weights], h0, dO
  * q, k ~ N(0,1), then each (token, head) row divided by its L2 norm in float64
    (workloads whose q/k pass through the short convolution are NOT normalised here:
    the layer core normalises after the convolution);
  * v, z, dO ~ N(0,1);
  * alpha = exp(-softplus(x) * 0.1), x ~ N(0,1)   (per key channel, or one per head);
  * b, w, beta = sigmoid(x), x ~ N(0,1);
  * conv weights ~ N(0, 0.02^2)  (standard deviation 0.02);
  * h0 ~ N(0, 0.1^2) where a workload has an initial state.
Draws are made in float32 (numpy's float32 normal generator), transformed in float64 and
cast a single time to bf16 (round-to-nearest-even, via torch) or kept in float32.

Workload sizes follow the pages: 128-wide heads, chunk 64 and 4K training length
(Gated DeltaNet-2 news item on zubnet.ai; Gated DeltaNet explainer «Protocole expérimental»),
16 key / 128 value heads and kernel-4 convolution for the GQA layer core (mkdocs chapter
«Gated DeltaNet», «Les projections d'entrée», «La convolution causale»).
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Optional

import numpy as np
import torch

SEED_BASE = 1000


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int                 # 1..5, seed = SEED_BASE + index
    B: int
    T: int
    Hk: int
    Hv: int
    dk: int
    dv: int
    alpha_per_channel: bool    # alpha in (0,1)^dk per token/head, else one scalar per token/head
    gates_per_channel: bool    # separate erase b (dk) and write w (dv); else scalar beta
    dtype: str                 # "bf16" | "f32"  (q, k, v, dO and outputs)
    gate_dtype: str            # "bf16" | "f32"  (alpha, b, w / beta)
    has_h0: bool
    conv: bool = False         # k=4 causal depthwise conv + SiLU (+ L2 on q,k) before the recurrence
    swish_gate: bool = False   # y = o * z * sigmoid(z) after the recurrence
    decode_steps: int = 0      # > 0: single-token decode workload, B = number of sequences
    chunk: int = 64

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def tokens(self) -> int:
        return self.B * (self.decode_steps if self.decode_steps else self.T)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("gdn2_fwd_tiny_f32", 1, B=1, T=256, Hk=2, Hv=2, dk=64, dv=64,
                 alpha_per_channel=True, gates_per_channel=True, dtype="f32", gate_dtype="f32",
                 has_h0=False),
        Workload("gdn_fwd_scalar_bf16", 2, B=8, T=4096, Hk=16, Hv=16, dk=128, dv=128,
                 alpha_per_channel=False, gates_per_channel=False, dtype="bf16", gate_dtype="f32",
                 has_h0=False),
        Workload("gdn2_fwd_bwd_bf16", 3, B=8, T=4096, Hk=16, Hv=16, dk=128, dv=128,
                 alpha_per_channel=True, gates_per_channel=True, dtype="bf16", gate_dtype="bf16",
                 has_h0=True),
        Workload("gqa_layer_core_bf16", 4, B=2, T=16384, Hk=16, Hv=128, dk=128, dv=128,
                 alpha_per_channel=False, gates_per_channel=False, dtype="bf16", gate_dtype="f32",
                 has_h0=False, conv=True, swish_gate=True),
        Workload("gdn2_decode_bf16", 5, B=256, T=1, Hk=16, Hv=16, dk=128, dv=128,
                 alpha_per_channel=True, gates_per_channel=True, dtype="bf16", gate_dtype="bf16",
                 has_h0=True, decode_steps=1024),
    ]
}


def _torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def _cast(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Single cast of a float array to the stated dtype (bf16 rounds to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(_torch_dtype(dtype)).contiguous()


def _normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _l2_rows(x: np.ndarray) -> np.ndarray:
    """Divide every last-axis row by its L2 norm, computed in float64 (input recipe)."""
    flat = x.reshape(-1, x.shape[-1])
    out = np.empty_like(flat)
    step = 1 << 18
    for i in range(0, flat.shape[0], step):
        blk = flat[i:i + step].astype(np.float64)
        nrm = np.sqrt(np.sum(blk * blk, axis=-1, keepdims=True))
        out[i:i + step] = (blk / nrm).astype(np.float32)
    return out.reshape(x.shape)


def _decay(x: np.ndarray, scale: float = 0.1) -> np.ndarray:
    """alpha = exp(-softplus(x) * scale), evaluated in float64 (input recipe: scale 0.1)."""
    x = x.astype(np.float64)
    sp = np.logaddexp(0.0, x)
    return np.exp(-scale * sp)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float64)
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def draw(B: int, T: int, Hk: int, Hv: int, dk: int, dv: int, *,
         alpha_per_channel: bool, gates_per_channel: bool, dtype: str = "bf16",
         gate_dtype: Optional[str] = None, seed: int = 0, has_h0: bool = True,
         conv: bool = False, swish_gate: bool = False, with_dout: bool = False,
         with_dht: bool = False, normalise_qk: Optional[bool] = None,
         erase_scale: float = 1.0, decay_scale: float = 0.1) -> Dict[str, object]:
    """Draw one batch of chunkwise-forward/backward inputs.

    decay_scale replaces the recipe's 0.1 in alpha = exp(-softplus(x) * 0.1): larger values give
    fast-forgetting gates (3 puts the typical alpha near 0.1 and the smallest near 1e-3), the range
    where a chunk's decay product leaves the chunk kernels' factorised range.

    erase_scale multiplies the erase gate b (or the scalar beta): 2 gives the negative-eigenvalue
    range b, beta in [0, 2] of the explainer's «Réunir les deux» note (the transition's eigenvalue
    along k is then 1 - beta in [-1, 1]); the write gate w stays in [0, 1].

    Returns a dict of torch CPU tensors in token-major layouts:
      q, k [B,T,Hk,dk]; v [B,T,Hv,dv]; alpha [B,T,Hv,dk] or [B,T,Hv];
      b [B,T,Hv,dk] and w [B,T,Hv,dv] (channel gates) or beta [B,T,Hv] (scalar);
      z [B,T,Hv,dv] (swish gate), conv_w [Hk*dk*2 + Hv*dv, 4] (conv), h0 [B,Hv,dk,dv] f32,
      dout [B,T,Hv,dv], dht [B,Hv,dk,dv] f32 — each only when requested.
    """
    gate_dtype = gate_dtype or dtype
    if normalise_qk is None:
        normalise_qk = not conv
    rng = np.random.default_rng(seed)
    out: Dict[str, object] = {}
    q = _normal(rng, (B, T, Hk, dk))
    k = _normal(rng, (B, T, Hk, dk))
    if normalise_qk:
        q = _l2_rows(q)
        k = _l2_rows(k)
    out["q"] = _cast(q, dtype)
    out["k"] = _cast(k, dtype)
    del q, k
    out["v"] = _cast(_normal(rng, (B, T, Hv, dv)), dtype)
    a_shape = (B, T, Hv, dk) if alpha_per_channel else (B, T, Hv)
    out["alpha"] = _cast(_decay(_normal(rng, a_shape), decay_scale), gate_dtype)
    if gates_per_channel:
        out["b"] = _cast(erase_scale * _sigmoid(_normal(rng, (B, T, Hv, dk))), gate_dtype)
        out["w"] = _cast(_sigmoid(_normal(rng, (B, T, Hv, dv))), gate_dtype)
    else:
        out["beta"] = _cast(erase_scale * _sigmoid(_normal(rng, (B, T, Hv))), gate_dtype)
    if swish_gate:
        out["z"] = _cast(_normal(rng, (B, T, Hv, dv)), dtype)
    if conv:
        cch = 2 * Hk * dk + Hv * dv
        out["conv_w"] = _cast(_normal(rng, (cch, 4), std=0.02), dtype)
    if has_h0:
        out["h0"] = torch.from_numpy(_normal(rng, (B, Hv, dk, dv), std=0.1))
    if with_dout:
        out["dout"] = _cast(_normal(rng, (B, T, Hv, dv)), dtype)
    if with_dht:
        out["dht"] = torch.from_numpy(_normal(rng, (B, Hv, dk, dv)))
    return out


def workload_inputs(name: str, *, with_dout: Optional[bool] = None, **size_overrides) -> Dict[str, object]:
    """Inputs of a named chunkwise workload (optionally at reduced sizes, same recipe)."""
    wl = WORKLOADS[name]
    if wl.decode_steps:
        raise ValueError("decode workloads are drawn step by step: use decode_inputs()")
    sizes = dict(B=wl.B, T=wl.T, Hk=wl.Hk, Hv=wl.Hv, dk=wl.dk, dv=wl.dv)
    sizes.update(size_overrides)
    if with_dout is None:
        with_dout = wl.index == 3
    return draw(**sizes, alpha_per_channel=wl.alpha_per_channel,
                gates_per_channel=wl.gates_per_channel, dtype=wl.dtype,
                gate_dtype=wl.gate_dtype, seed=wl.seed, has_h0=wl.has_h0, conv=wl.conv,
                swish_gate=wl.swish_gate, with_dout=with_dout)


def decode_initial_state(name: str = "gdn2_decode_bf16", **size_overrides) -> torch.Tensor:
    """Initial fp32 state [N,Hv,dk,dv] ~ N(0, 0.1^2) of a decode workload."""
    wl = WORKLOADS[name]
    N = size_overrides.get("B", wl.B)
    Hv = size_overrides.get("Hv", wl.Hv)
    dk = size_overrides.get("dk", wl.dk)
    dv = size_overrides.get("dv", wl.dv)
    rng = np.random.default_rng(wl.seed)
    return torch.from_numpy(_normal(rng, (N, Hv, dk, dv), std=0.1))


def decode_step_inputs(name: str, step: int, **size_overrides) -> Dict[str, torch.Tensor]:
    """Per-step decode inputs, drawn from ``default_rng([seed, step])``.

    q, k [N,Hk,dk] (L2-normalised); v [N,Hv,dv]; alpha [N,Hv,dk] or [N,Hv];
    b [N,Hv,dk] and w [N,Hv,dv], or beta [N,Hv].
    """
    wl = WORKLOADS[name]
    N = size_overrides.get("B", wl.B)
    Hk = size_overrides.get("Hk", wl.Hk)
    Hv = size_overrides.get("Hv", wl.Hv)
    dk = size_overrides.get("dk", wl.dk)
    dv = size_overrides.get("dv", wl.dv)
    apc = size_overrides.get("alpha_per_channel", wl.alpha_per_channel)
    gpc = size_overrides.get("gates_per_channel", wl.gates_per_channel)
    rng = np.random.default_rng([wl.seed, step])
    out: Dict[str, torch.Tensor] = {}
    out["q"] = _cast(_l2_rows(_normal(rng, (N, Hk, dk))), wl.dtype)
    out["k"] = _cast(_l2_rows(_normal(rng, (N, Hk, dk))), wl.dtype)
    out["v"] = _cast(_normal(rng, (N, Hv, dv)), wl.dtype)
    out["alpha"] = _cast(_decay(_normal(rng, (N, Hv, dk) if apc else (N, Hv))), wl.gate_dtype)
    if gpc:
        out["b"] = _cast(_sigmoid(_normal(rng, (N, Hv, dk))), wl.gate_dtype)
        out["w"] = _cast(_sigmoid(_normal(rng, (N, Hv, dv))), wl.gate_dtype)
    else:
        out["beta"] = _cast(_sigmoid(_normal(rng, (N, Hv))), wl.gate_dtype)
    return out


def decode_inputs(name: str = "gdn2_decode_bf16", steps: Optional[int] = None, *,
                  threads: int = 8, **size_overrides) -> Dict[str, torch.Tensor]:
    """All steps of a decode workload stacked on a leading step axis ([steps, N, ...])."""
    wl = WORKLOADS[name]
    steps = wl.decode_steps if steps is None else steps
    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        per = list(ex.map(lambda s: decode_step_inputs(name, s, **size_overrides), range(steps)))
    return {key: torch.stack([p[key] for p in per]) for key in per[0]}
