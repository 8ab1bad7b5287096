"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

Every check here runs on the CPU (no GPU marker).  Each one is chosen so that a plausible
mistake in the oracle (a dropped term, a wrong sign or index, decay applied after the write,
erasing along the gated key instead of the key, a transposed operand, a lost scale, a wrong
GQA group) fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_inputs(rng, B, T, Hk, Hv, dk, dv, *, channel_alpha=True, channel_gates=True,
                h0=True, unit_keys=True):
    q = rng.standard_normal((B, T, Hk, dk))
    k = rng.standard_normal((B, T, Hk, dk))
    if unit_keys:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, Hv, dv))
    a_shape = (B, T, Hv, dk) if channel_alpha else (B, T, Hv)
    alpha = np.exp(-0.1 * np.logaddexp(0.0, rng.standard_normal(a_shape)))
    out = dict(q=q, k=k, v=v, alpha=alpha)
    if channel_gates:
        out["b"] = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv, dk))))
        out["w"] = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv, dv))))
    else:
        out["beta"] = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv))))
    if h0:
        out["h0"] = 0.3 * rng.standard_normal((B, Hv, dk, dv))
    return out


def relerr(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# --------------------------------------------------------------------------------------------
# Printed worked example: Gated DeltaNet explainer, «Trois règles, un même calcul».
# --------------------------------------------------------------------------------------------
def test_worked_example_three_rules():
    with open(os.path.join(GOLDEN, "worked_example_three_rules.json")) as f:
        g = json.load(f)
    keys = {n: np.array(v, dtype=float) for n, v in g["keys"].items()}
    T = len(g["writes"])
    k = np.stack([keys[n] for n, _ in g["writes"]])[None, :, None, :]
    v = np.array([val for _, val in g["writes"]], dtype=float)[None, :, None, None]
    for rule in g["rules"]:
        alpha = np.full((1, T, 1, 3), rule["alpha"])
        b = np.full((1, T, 1, 3), rule["b"])
        w = np.full((1, T, 1, 1), rule["w"])
        for name, expect in (("k1", rule["read_k1"]), ("k2", rule["read_k2"])):
            # Read through the readout path: query the last state with the key.
            q = np.zeros((1, T, 1, 3))
            q[0, -1, 0] = keys[name]
            o, hT = oracle.fwd(q, k, v, alpha, b=b, w=w)
            assert o[0, -1, 0, 0] == pytest.approx(expect, abs=1e-12), rule["name"]
            # And directly from the final state: S^T k.
            assert float((hT[0, 0].T @ keys[name])[0]) == pytest.approx(expect, abs=1e-12)


# --------------------------------------------------------------------------------------------
# Reductions (GDN-2 summary, end of «Règle Delta Portée-2»; explainer «Réunir les deux»,
# «DeltaNet : ne corriger que l'entrée visée»).
# --------------------------------------------------------------------------------------------
def _gdn_transposed(q, k, v, alpha, beta, h0):
    """Gated DeltaNet as the explainer writes it, state S' in R^{dv x dk}:
    S'_t = S'_{t-1} (alpha_t (I - beta_t k_t k_t^T)) + beta_t v_t k_t^T,  o_t = S'_t q_t."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    o = np.zeros((B, T, Hv, dv))
    hT = np.zeros((B, Hv, dk, dv))
    for b_ in range(B):
        for h in range(Hv):
            hk = h // (Hv // Hk)
            S = h0[b_, h].T.copy()
            for t in range(T):
                kk = k[b_, t, hk]
                M = alpha[b_, t, h] * (np.eye(dk) - beta[b_, t, h] * np.outer(kk, kk))
                S = S @ M + beta[b_, t, h] * np.outer(v[b_, t, h], kk)
                o[b_, t, h] = S @ q[b_, t, hk]
            hT[b_, h] = S.T
    return o, hT


def test_reduction_to_gated_deltanet():
    rng = np.random.default_rng(11)
    x = rand_inputs(rng, 2, 37, 2, 4, 8, 6, channel_alpha=False, channel_gates=False)
    o, hT = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], beta=x["beta"], h0=x["h0"])
    o_ref, hT_ref = _gdn_transposed(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["h0"])
    assert relerr(o, o_ref) < 1e-12
    assert relerr(hT, hT_ref) < 1e-12
    # Channel-wise code path with every channel equal to the scalar gives the same thing.
    B, T, Hv = x["alpha"].shape
    dk, dv = 8, 6
    o2, hT2 = oracle.fwd(x["q"], x["k"], x["v"],
                         np.repeat(x["alpha"][..., None], dk, -1),
                         b=np.repeat(x["beta"][..., None], dk, -1),
                         w=np.repeat(x["beta"][..., None], dv, -1), h0=x["h0"])
    assert relerr(o2, o_ref) < 1e-12
    assert relerr(hT2, hT_ref) < 1e-12


def test_reduction_to_deltanet():
    """alpha = 1: v_old = S' k, v_new = beta v + (1 - beta) v_old, S' += (v_new - v_old) k^T."""
    rng = np.random.default_rng(12)
    x = rand_inputs(rng, 1, 29, 1, 1, 7, 5, channel_alpha=False, channel_gates=False)
    ones = np.ones_like(x["alpha"])
    o, hT = oracle.fwd(x["q"], x["k"], x["v"], ones, beta=x["beta"], h0=x["h0"])
    S = x["h0"][0, 0].T.copy()
    for t in range(29):
        kk, beta = x["k"][0, t, 0], x["beta"][0, t, 0]
        v_old = S @ kk
        v_new = beta * x["v"][0, t, 0] + (1 - beta) * v_old
        S = S - np.outer(v_old, kk) + np.outer(v_new, kk)
        assert np.allclose(o[0, t, 0], S @ x["q"][0, t, 0], rtol=0, atol=1e-12)
    assert relerr(hT[0, 0], S.T) < 1e-12


def test_linear_attention_closed_form():
    """alpha = 1, b = 0, w = 1: O = ((Q K^T) * causal mask) V, times the scale."""
    rng = np.random.default_rng(13)
    x = rand_inputs(rng, 1, 50, 1, 1, 9, 4, h0=False)
    T = 50
    one_a = np.ones((1, T, 1, 9))
    zero_b = np.zeros((1, T, 1, 9))
    one_w = np.ones((1, T, 1, 4))
    o, hT = oracle.fwd(x["q"], x["k"], x["v"], one_a, b=zero_b, w=one_w, scale=0.7)
    Q, K, V = x["q"][0, :, 0], x["k"][0, :, 0], x["v"][0, :, 0]
    o_ref = 0.7 * (np.tril(Q @ K.T) @ V)
    assert relerr(o[0, :, 0], o_ref) < 1e-12
    assert relerr(hT[0, 0], K.T @ V) < 1e-12


def test_decay_only_closed_form():
    """b = 0, w = 1 (Mamba-2 style, channel-wise decay):
    o_t[j] = sum_{s<=t} sum_c q_t[c] k_s[c] prod_{s<i<=t} alpha_i[c] v_s[j]  (+ decayed h0)."""
    rng = np.random.default_rng(14)
    x = rand_inputs(rng, 1, 40, 1, 1, 6, 5)
    T, dk, dv = 40, 6, 5
    o, hT = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], b=np.zeros((1, T, 1, dk)),
                       w=np.ones((1, T, 1, dv)), h0=x["h0"])
    L = np.cumsum(np.log(x["alpha"][0, :, 0]), axis=0)  # [T, dk] inclusive
    Q, K, V, S0 = x["q"][0, :, 0], x["k"][0, :, 0], x["v"][0, :, 0], x["h0"][0, 0]
    o_ref = np.zeros((T, dv))
    for t in range(T):
        for s in range(t + 1):
            o_ref[t] += np.sum(Q[t] * K[s] * np.exp(L[t] - L[s])) * V[s]
        o_ref[t] += (Q[t] * np.exp(L[t])) @ S0
    assert relerr(o[0, :, 0], o_ref) < 1e-12


# --------------------------------------------------------------------------------------------
# Invariants of one GDN-2 step.
# --------------------------------------------------------------------------------------------
def _one_step(rng, dk=7, dv=5):
    x = rand_inputs(rng, 1, 1, 1, 1, dk, dv)
    o, hT = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"])
    return x, hT[0, 0]


def test_exact_recall_unit_key():
    """Unit key, b = w = 1, alpha = 1: reading the new state at k_t returns v_t exactly
    (explainer, Figure 1 caption remark and «DeltaNet»)."""
    rng = np.random.default_rng(15)
    B, T, dk, dv = 2, 33, 8, 6
    x = rand_inputs(rng, B, T, 1, 1, dk, dv)
    o, _ = oracle.fwd(x["k"], x["k"], x["v"], np.ones((B, T, 1, dk)), b=np.ones((B, T, 1, dk)),
                      w=np.ones((B, T, 1, dv)), h0=x["h0"])
    assert np.max(np.abs(o - x["v"])) < 1e-12


def test_edit_invariant():
    """S_t^T e_t = (1 - kappa) Sbar^T e_t + kappa z_t with kappa = k_t . e_t
    (GDN-2 summary, §2 «Perspective de Mise à Jour des Poids Rapides»: the step moves the read
    at e_t toward the gated target z_t)."""
    rng = np.random.default_rng(16)
    for _ in range(5):
        x, S = _one_step(rng)
        k, b_, w_ = x["k"][0, 0, 0], x["b"][0, 0, 0], x["w"][0, 0, 0]
        e = b_ * k
        z = w_ * x["v"][0, 0, 0]
        Sbar = x["alpha"][0, 0, 0][:, None] * x["h0"][0, 0]
        kappa = k @ e
        assert np.allclose(S.T @ e, (1 - kappa) * (Sbar.T @ e) + kappa * z, atol=1e-13)


def test_reflection_at_beta_two_is_an_involution():
    """Negative-eigenvalue range (explainer, «Réunir les deux», note on beta in [0, 2]): with
    alpha = 1, a unit key, beta = 2 and no write (v = 0) the step is the Householder reflection
    S -> (I - 2 k k^T) S, so the same step twice returns the state, and once negates the read
    at k while sparing every direction orthogonal to k."""
    rng = np.random.default_rng(31)
    dk, dv = 6, 5
    k = rng.standard_normal(dk)
    k /= np.linalg.norm(k)
    h0 = rng.standard_normal((1, 1, dk, dv))
    kk = np.broadcast_to(k, (1, 2, 1, dk)).copy()
    ones = np.ones((1, 2, 1))
    v0 = np.zeros((1, 2, 1, dv))
    _, once = oracle.fwd(kk[:, :1], kk[:, :1], v0[:, :1], ones[:, :1], beta=2 * ones[:, :1], h0=h0)
    _, twice = oracle.fwd(kk, kk, v0, ones, beta=2 * ones, h0=h0)
    assert np.allclose(twice[0, 0], h0[0, 0], atol=1e-13)
    assert np.allclose(once[0, 0].T @ k, -(h0[0, 0].T @ k), atol=1e-13)
    u = rng.standard_normal(dk)
    u -= (u @ k) * k
    assert np.allclose(u @ once[0, 0], u @ h0[0, 0], atol=1e-13)


def test_edit_invariant_over_the_negative_eigenvalue_range():
    """The edit invariant S_t^T e_t = (1 - kappa) Sbar^T e_t + kappa z_t holds unchanged for erase
    gates b in [0, 2] (kappa = k . e up to 2 for a unit key)."""
    rng = np.random.default_rng(32)
    for _ in range(5):
        x = rand_inputs(rng, 1, 1, 1, 1, 7, 5)
        x["b"] = 2.0 * x["b"]
        _, hT = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"])
        k, b_, w_ = x["k"][0, 0, 0], x["b"][0, 0, 0], x["w"][0, 0, 0]
        e, z = b_ * k, w_ * x["v"][0, 0, 0]
        Sbar = x["alpha"][0, 0, 0][:, None] * x["h0"][0, 0]
        kappa = k @ e
        assert np.allclose(hT[0, 0].T @ e, (1 - kappa) * (Sbar.T @ e) + kappa * z, atol=1e-13)


def test_orthogonal_keys_spared():
    """For u orthogonal to k_t: u^T S_t = u^T D_t S_{t-1} (explainer, «DeltaNet»)."""
    rng = np.random.default_rng(17)
    for _ in range(5):
        x, S = _one_step(rng)
        k = x["k"][0, 0, 0]
        u = rng.standard_normal(k.shape)
        u -= (u @ k) * k
        Sbar = x["alpha"][0, 0, 0][:, None] * x["h0"][0, 0]
        assert np.allclose(u @ S, u @ Sbar, atol=1e-13)
        # The direction k_t itself does change (the pin above is not vacuous).
        assert not np.allclose(k @ S, k @ Sbar, atol=1e-6)


def test_gqa_equals_replicated_heads():
    """A value head reads the key head head_map[hv]; replicating q/k per value head with an
    identity map must give the same result."""
    rng = np.random.default_rng(18)
    x = rand_inputs(rng, 2, 21, 2, 6, 5, 4)
    hmap = np.array([1, 0, 1, 0, 0, 1], dtype=np.int32)
    o, hT = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"],
                       head_map=hmap)
    qr, kr = x["q"][:, :, hmap], x["k"][:, :, hmap]
    o2, hT2 = oracle.fwd(qr, kr, x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"],
                         head_map=np.arange(6))
    assert np.array_equal(o, o2) and np.array_equal(hT, hT2)


# --------------------------------------------------------------------------------------------
# Chunkwise form == sequential form (explainer «Rendre l'entraînement parallèle»; GDN-2
# summary §3).
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("C", [8, 16, 64])
@pytest.mark.parametrize("channel", [True, False])
def test_chunk_form_matches_sequential(C, channel):
    rng = np.random.default_rng(19 + C)
    x = rand_inputs(rng, 2, 100, 1, 2, 8, 6, channel_alpha=channel, channel_gates=channel)
    kw = dict(b=x.get("b"), w=x.get("w"), beta=x.get("beta"), h0=x["h0"], scale=0.9)
    o, hT = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], **kw)
    oc, hTc = oracle.chunk_fwd(x["q"], x["k"], x["v"], x["alpha"], C=C, **kw)
    assert relerr(oc, o) < 1e-12
    assert relerr(hTc, hT) < 1e-12


# --------------------------------------------------------------------------------------------
# Carry: split sequences and decode steps.
# --------------------------------------------------------------------------------------------
def test_split_sequence_carry():
    rng = np.random.default_rng(20)
    x = rand_inputs(rng, 2, 45, 1, 2, 6, 5)
    o, hT = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"])
    cut = 17
    part = lambda a, sl: a[:, sl]
    o1, h1 = oracle.fwd(*(part(x[n], slice(0, cut)) for n in ("q", "k", "v", "alpha")),
                        b=x["b"][:, :cut], w=x["w"][:, :cut], h0=x["h0"])
    o2, h2 = oracle.fwd(*(part(x[n], slice(cut, None)) for n in ("q", "k", "v", "alpha")),
                        b=x["b"][:, cut:], w=x["w"][:, cut:], h0=h1)
    assert relerr(np.concatenate([o1, o2], axis=1), o) < 1e-13
    assert relerr(h2, hT) < 1e-13


def test_decode_steps_equal_forward():
    rng = np.random.default_rng(21)
    x = rand_inputs(rng, 3, 12, 1, 2, 6, 5)
    o, hT = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"], scale=1.3)
    S = x["h0"]
    for t in range(12):
        ot, S = oracle.decode_step(S, x["q"][:, t], x["k"][:, t], x["v"][:, t], x["alpha"][:, t],
                                   b=x["b"][:, t], w=x["w"][:, t], scale=1.3)
        assert relerr(ot, o[:, t]) < 1e-13
    assert relerr(S, hT) < 1e-13


# --------------------------------------------------------------------------------------------
# Backward: central finite differences of the oracle's own forward.
# --------------------------------------------------------------------------------------------
def _fd_check(x, kw_mode, T, dout, dht, scale):
    names = ["q", "k", "v", "alpha"] + kw_mode + ["h0"]

    def loss(vals):
        kw = {n: vals[n] for n in kw_mode}
        o, hT = oracle.fwd(vals["q"], vals["k"], vals["v"], vals["alpha"], h0=vals["h0"],
                           scale=scale, nthreads=1, **kw)
        return np.sum(o * dout) + np.sum(hT * dht)

    kw = {n: x[n] for n in kw_mode}
    g = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"], scale=scale, dout=dout,
                   dht=dht, nthreads=1, **kw)
    key = {"q": "dq", "k": "dk", "v": "dv", "alpha": "dalpha", "b": "db", "w": "dw",
           "beta": "dbeta", "h0": "dh0"}
    h = 1e-6
    for n in names:
        base = x[n]
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = {m: x[m].copy() for m in names}
            minus = {m: x[m].copy() for m in names}
            plus[n][idx] += h
            minus[n][idx] -= h
            fd[idx] = (loss(plus) - loss(minus)) / (2 * h)
        an = g[key[n]]
        err = np.max(np.abs(an - fd)) / max(np.max(np.abs(fd)), 1e-12)
        assert err < 1e-6, (n, err)


@pytest.mark.parametrize("mode", ["gdn2", "gdn", "kda"])
def test_backward_finite_differences(mode):
    rng = np.random.default_rng({"gdn2": 31, "gdn": 32, "kda": 33}[mode])
    B, T, Hk, Hv, dk, dv = 1, 9, 1, 2, 4, 3
    x = rand_inputs(rng, B, T, Hk, Hv, dk, dv, channel_alpha=(mode != "gdn"),
                    channel_gates=(mode == "gdn2"))
    kw_mode = ["b", "w"] if mode == "gdn2" else ["beta"]
    dout = rng.standard_normal((B, T, Hv, dv))
    dht = rng.standard_normal((B, Hv, dk, dv))
    _fd_check(x, kw_mode, T, dout, dht, scale=0.8)


def test_backward_crosses_checkpoint_segments():
    """T > 64 exercises the oracle's segment recomputation (gradients checked on a few entries
    of every input, including ones before and after the segment boundary)."""
    rng = np.random.default_rng(34)
    B, T, Hk, Hv, dk, dv = 1, 70, 1, 1, 3, 2
    x = rand_inputs(rng, B, T, Hk, Hv, dk, dv)
    dout = rng.standard_normal((B, T, Hv, dv))
    dht = rng.standard_normal((B, Hv, dk, dv))
    g = oracle.bwd(x["q"], x["k"], x["v"], x["alpha"], b=x["b"], w=x["w"], h0=x["h0"],
                   dout=dout, dht=dht, nthreads=1)

    def loss(vals):
        o, hT = oracle.fwd(vals["q"], vals["k"], vals["v"], vals["alpha"], b=vals["b"],
                           w=vals["w"], h0=vals["h0"], nthreads=1)
        return np.sum(o * dout) + np.sum(hT * dht)

    h = 1e-6
    key = {"q": "dq", "k": "dk", "v": "dv", "alpha": "dalpha", "b": "db", "w": "dw"}
    for n in key:
        for t in (0, 5, 63, 64, 69):
            for c in range(x[n].shape[-1]):
                idx = (0, t, 0, c)
                p = {m: x[m].copy() for m in x}
                mi = {m: x[m].copy() for m in x}
                p[n][idx] += h
                mi[n][idx] -= h
                fd = (loss(p) - loss(mi)) / (2 * h)
                assert abs(g[key[n]][idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (n, idx)


# --------------------------------------------------------------------------------------------
# Layer-core pieces: short convolution, L2 norm, swish gate (explainer Figure 1 caption;
# mkdocs chapter «La convolution causale», «La porte de sortie»).
# --------------------------------------------------------------------------------------------
def test_conv_matches_library_convolution_and_carries_history():
    rng = np.random.default_rng(40)
    B, T, C = 2, 23, 5
    x = rng.standard_normal((B, T, C))
    w = rng.standard_normal((C, 4))
    y, hist = oracle.conv_silu(x, w)
    for b_ in range(B):
        for c in range(C):
            # Causal conv: numpy's full convolution with the reversed taps, first T outputs.
            pre = np.convolve(x[b_, :, c], w[c, ::-1])[:T]
            assert np.allclose(y[b_, :, c], pre / (1 + np.exp(-pre)), atol=1e-13)
    assert np.array_equal(hist, np.transpose(x[:, -3:, :], (0, 2, 1)))
    # Two calls with the carried history equal one call.
    y1, h1 = oracle.conv_silu(x[:, :10], w)
    y2, h2 = oracle.conv_silu(x[:, 10:], w, hist=h1)
    assert np.allclose(np.concatenate([y1, y2], 1), y, atol=1e-14)
    assert np.array_equal(h2, hist)


def test_l2norm_and_swish_gate():
    rng = np.random.default_rng(41)
    x = rng.standard_normal((7, 16)) * 3
    y = oracle.l2norm(x, eps=0.0)
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-14)
    assert np.allclose(y * np.linalg.norm(x, axis=-1, keepdims=True), x, atol=1e-13)
    o = rng.standard_normal(100)
    z = rng.standard_normal(100) * 4
    from scipy.special import expit
    assert np.allclose(oracle.swish_gate(o, z), o * z * expit(z), atol=1e-14)


@pytest.mark.parametrize("channel_gates", [False, True])
def test_layer_backward_finite_differences(channel_gates):
    """The layer core's reverse mode (conv k=4, SiLU, L2 norm, the recurrence, the swish gate)
    against central differences of sum(y * dy) + sum(hT * dht), for every input, on a tiny GQA
    layer.  The forward here is composed from the oracle's own conv_silu / l2norm / fwd /
    swish_gate, so the pin ties the hand-written reverse steps to their forward definitions."""
    rng = np.random.default_rng(55)
    B, T, Hk, Hv, d = 1, 6, 1, 2, 4
    cq = Hk * d
    x = dict(xq=rng.standard_normal((B, T, Hk, d)), xk=rng.standard_normal((B, T, Hk, d)),
             xv=rng.standard_normal((B, T, Hv, d)), conv_w=0.5 * rng.standard_normal((2 * cq + Hv * d, 4)),
             alpha=np.exp(-0.1 * np.logaddexp(0.0, rng.standard_normal((B, T, Hv)))),
             z=rng.standard_normal((B, T, Hv, d)), h0=0.3 * rng.standard_normal((B, Hv, d, d)))
    if channel_gates:
        x["b"] = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv, d))))
        x["w"] = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv, d))))
        gnames = ["b", "w"]
    else:
        x["beta"] = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv))))
        gnames = ["beta"]
    dy = rng.standard_normal((B, T, Hv, d))
    dht = rng.standard_normal((B, Hv, d, d))
    scale = 0.8

    def loss(vals):
        W = vals["conv_w"]
        q, _ = oracle.conv_silu(vals["xq"].reshape(B, T, cq), W[:cq])
        k, _ = oracle.conv_silu(vals["xk"].reshape(B, T, cq), W[cq:2 * cq])
        v, _ = oracle.conv_silu(vals["xv"].reshape(B, T, Hv * d), W[2 * cq:])
        q = oracle.l2norm(q.reshape(B, T, Hk, d))
        k = oracle.l2norm(k.reshape(B, T, Hk, d))
        o, hT = oracle.fwd(q, k, v.reshape(B, T, Hv, d), vals["alpha"], h0=vals["h0"], scale=scale,
                           nthreads=1, **{n: vals[n] for n in gnames})
        return np.sum(oracle.swish_gate(o, vals["z"]) * dy) + np.sum(hT * dht)

    g = oracle.layer_core_bwd(x["xq"], x["xk"], x["xv"], x["conv_w"], x["alpha"], x["z"], dy, h0=x["h0"],
                              dht=dht, scale=scale, **{n: x[n] for n in gnames})
    key = {"xq": "dxq", "xk": "dxk", "xv": "dxv", "conv_w": "dconv_w", "alpha": "dalpha", "z": "dz",
           "h0": "dh0", "b": "db", "w": "dw", "beta": "dbeta"}
    names = list(x)
    h = 1e-6
    for n in names:
        base = x[n]
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = {m: x[m].copy() for m in names}
            minus = {m: x[m].copy() for m in names}
            plus[n][idx] += h
            minus[n][idx] -= h
            fd[idx] = (loss(plus) - loss(minus)) / (2 * h)
        err = np.max(np.abs(g[key[n]] - fd)) / max(np.max(np.abs(fd)), 1e-12)
        assert err < 1e-6, (n, err)


# ---- segment maps (sequence split along time) --------------------------------------------------
def _gates(x):
    return dict(beta=x["beta"]) if "beta" in x else dict(b=x["b"], w=x["w"])


@pytest.mark.parametrize("channel", [True, False])
def test_segment_map_is_the_state_map(channel):
    """M S + N equals the recurrence run from S, for any entering state S (the update is affine in
    the state): checked against fwd() from two random states."""
    rng = np.random.default_rng(71)
    x = rand_inputs(rng, 2, 37, 1, 2, 8, 8, channel_alpha=channel, channel_gates=channel, h0=False)
    M, N = oracle.segment_map(x["q"], x["k"], x["v"], x["alpha"], **_gates(x))
    for _ in range(2):
        S = rng.standard_normal((2, 2, 8, 8))
        _, hT = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], h0=S, **_gates(x))
        assert relerr(oracle.compose(M, N, S), hT) < 1e-12


def test_segment_maps_compose_over_a_split_sequence():
    """Two segments: (M2 M1, M2 N1 + N2) is the map of the whole, and the exclusive composition
    gives the state entering the second segment."""
    rng = np.random.default_rng(72)
    x = rand_inputs(rng, 1, 50, 2, 4, 8, 8, h0=True)
    cut = 21
    seg = lambda lo, hi: {k: (v[:, lo:hi] if v.ndim >= 3 and k != "h0" else v) for k, v in x.items()}
    a, b = seg(0, cut), seg(cut, 50)
    M1, N1 = oracle.segment_map(a["q"], a["k"], a["v"], a["alpha"], **_gates(a))
    M2, N2 = oracle.segment_map(b["q"], b["k"], b["v"], b["alpha"], **_gates(b))
    M, N = oracle.segment_map(x["q"], x["k"], x["v"], x["alpha"], **_gates(x))
    assert relerr(np.einsum("bhij,bhjk->bhik", M2, M1), M) < 1e-12
    assert relerr(oracle.compose(M2, N2, N1), N) < 1e-12
    _, h_mid = oracle.fwd(a["q"], a["k"], a["v"], a["alpha"], h0=x["h0"], **_gates(a))
    assert relerr(oracle.compose(M1, N1, x["h0"]), h_mid) < 1e-12


def test_segment_map_closed_forms():
    """No erase (b = 0): M = Diag(prod alpha) (decay only), N = sum_t (prod_{s>t} alpha_s) k_t z_t^T;
    with alpha = 1 as well, M = I and N = K^T Z (linear attention's running sum)."""
    rng = np.random.default_rng(73)
    x = rand_inputs(rng, 1, 30, 1, 1, 6, 6, h0=False)
    x["b"] = np.zeros_like(x["b"])
    M, N = oracle.segment_map(x["q"], x["k"], x["v"], x["alpha"], **_gates(x))
    a = x["alpha"][0, :, 0]                      # [T, dk]
    assert relerr(M[0, 0], np.diag(np.prod(a, axis=0))) < 1e-14
    tail = np.array([np.prod(a[t + 1:], axis=0) for t in range(30)])  # [T, dk]
    z = x["w"][0, :, 0] * x["v"][0, :, 0]
    N_ref = np.einsum("tc,tc,tj->cj", tail, x["k"][0, :, 0], z)
    assert relerr(N[0, 0], N_ref) < 1e-12
    x["alpha"] = np.ones_like(x["alpha"])
    M, N = oracle.segment_map(x["q"], x["k"], x["v"], x["alpha"], **_gates(x))
    assert np.array_equal(M[0, 0], np.eye(6))
    assert relerr(N[0, 0], x["k"][0, :, 0].T @ z) < 1e-12


def test_transposed_composition_carries_a_state_gradient_back():
    """For L = <G, S_out> with S_out = M S_in + N, dL/dS_in = M^T G: the transposed composition,
    checked by finite differences of the oracle's own forward."""
    rng = np.random.default_rng(74)
    x = rand_inputs(rng, 1, 12, 1, 1, 4, 4, h0=True)
    M, N = oracle.segment_map(x["q"], x["k"], x["v"], x["alpha"], **_gates(x))
    G = rng.standard_normal((1, 1, 4, 4))
    grad = oracle.compose(M, np.zeros_like(G), G, transpose=True)
    eps = 1e-6
    for (i, j) in [(0, 0), (1, 3), (3, 2)]:
        d = np.zeros_like(x["h0"])
        d[0, 0, i, j] = eps
        _, hp = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"] + d, **_gates(x))
        _, hm = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], h0=x["h0"] - d, **_gates(x))
        fd = np.sum(G * (hp - hm)) / (2 * eps)
        assert abs(fd - grad[0, 0, i, j]) < 1e-7 * max(1.0, abs(fd))


# ---- the layer's output norm ---------------------------------------------------------------------
def test_gated_rmsnorm_matches_the_library_rms_norm():
    """oracle.gated_rmsnorm against torch's own rms_norm (a library routine, float64) times
    swish(z); and invariance of the normalised rows to a positive scale of o."""
    import torch
    rng = np.random.default_rng(75)
    o = rng.standard_normal((2, 5, 3, 16))
    z = rng.standard_normal((2, 5, 3, 16))
    wn = rng.standard_normal(16)
    y = oracle.gated_rmsnorm(o, z, wn)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(o), (16,), weight=torch.from_numpy(wn), eps=oracle.RMS_EPS)
    ref = ref.numpy() * z / (1.0 + np.exp(-z))
    assert relerr(y, ref) < 1e-13
    assert relerr(oracle.gated_rmsnorm(7.5 * o, z, wn), y) < 1e-6


def test_layer_backward_with_output_norm_finite_differences():
    """The layer core with its output norm (y = RMSNorm(o) * norm_w * swish(z)): every gradient,
    norm_w's included, against central differences of sum(y * dy) + sum(hT * dht)."""
    rng = np.random.default_rng(76)
    B, T, Hk, Hv, d = 1, 5, 1, 2, 4
    cq = Hk * d
    x = dict(xq=rng.standard_normal((B, T, Hk, d)), xk=rng.standard_normal((B, T, Hk, d)),
             xv=rng.standard_normal((B, T, Hv, d)), conv_w=0.5 * rng.standard_normal((2 * cq + Hv * d, 4)),
             alpha=np.exp(-0.1 * np.logaddexp(0.0, rng.standard_normal((B, T, Hv)))),
             beta=1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv)))),
             z=rng.standard_normal((B, T, Hv, d)), h0=0.3 * rng.standard_normal((B, Hv, d, d)),
             norm_w=rng.standard_normal(d))
    dy = rng.standard_normal((B, T, Hv, d))
    dht = rng.standard_normal((B, Hv, d, d))

    def loss(vals):
        W = vals["conv_w"]
        q, _ = oracle.conv_silu(vals["xq"].reshape(B, T, cq), W[:cq])
        k, _ = oracle.conv_silu(vals["xk"].reshape(B, T, cq), W[cq:2 * cq])
        v, _ = oracle.conv_silu(vals["xv"].reshape(B, T, Hv * d), W[2 * cq:])
        q = oracle.l2norm(q.reshape(B, T, Hk, d))
        k = oracle.l2norm(k.reshape(B, T, Hk, d))
        o, hT = oracle.fwd(q, k, v.reshape(B, T, Hv, d), vals["alpha"], beta=vals["beta"], h0=vals["h0"],
                           nthreads=1)
        return np.sum(oracle.gated_rmsnorm(o, vals["z"], vals["norm_w"]) * dy) + np.sum(hT * dht)

    g = oracle.layer_core_bwd(x["xq"], x["xk"], x["xv"], x["conv_w"], x["alpha"], x["z"], dy, beta=x["beta"],
                              h0=x["h0"], dht=dht, norm_w=x["norm_w"])
    key = {"xq": "dxq", "xk": "dxk", "xv": "dxv", "conv_w": "dconv_w", "alpha": "dalpha", "z": "dz",
           "h0": "dh0", "beta": "dbeta", "norm_w": "dnorm_w"}
    h = 1e-6
    for n in x:
        fd = np.zeros_like(x[n])
        it = np.nditer(x[n], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = {m: x[m].copy() for m in x}
            minus = {m: x[m].copy() for m in x}
            plus[n][idx] += h
            minus[n][idx] -= h
            fd[idx] = (loss(plus) - loss(minus)) / (2 * h)
        err = np.max(np.abs(g[key[n]] - fd)) / max(np.max(np.abs(fd)), 1e-12)
        assert err < 1e-6, (n, err)


# ---- gates from logits -----------------------------------------------------------------------------
def test_gates_from_logits_closed_forms():
    """alpha = exp(-a softplus(x)): at x = 0 it is 2^-a; a = 0.1 is the input recipe's decay; the
    sigmoid gates are 1/2 at 0 and symmetric."""
    x = np.zeros((1, 2, 3, 4))
    a, b, w, _ = oracle.gates_from_logits(x, np.array([0.1, 1.0, 2.0]), x_b=x, x_w=-x)
    assert np.allclose(a[0, 0, :, 0], [2 ** -0.1, 0.5, 0.25], rtol=0, atol=1e-15)
    assert np.all(b == 0.5) and np.all(w == 0.5)
    rng = np.random.default_rng(77)
    xr = rng.standard_normal((2, 3, 4))
    _, _, _, beta = oracle.gates_from_logits(xr, np.ones(4), x_beta=xr)
    _, _, _, beta_m = oracle.gates_from_logits(xr, np.ones(4), x_beta=-xr)
    assert np.allclose(beta + beta_m, 1.0, atol=1e-15)


@pytest.mark.parametrize("channel", [True, False])
def test_logit_gradients_finite_differences(channel):
    """The recurrence's gradients pushed through the gate functions, against central differences of
    a loss of the outputs computed from the logits."""
    rng = np.random.default_rng(78)
    B, T, Hk, Hv, d = 1, 7, 1, 2, 4
    x = rand_inputs(rng, B, T, Hk, Hv, d, d, channel_alpha=channel, channel_gates=channel, h0=True)
    xa = rng.standard_normal(x["alpha"].shape)
    a_scale = np.array([0.3, 1.7])
    lg = {"x_b": rng.standard_normal(x["b"].shape), "x_w": rng.standard_normal(x["w"].shape)} if channel else \
         {"x_beta": rng.standard_normal(x["beta"].shape)}
    dout = rng.standard_normal((B, T, Hv, d))

    def loss(xa_, a_, lg_):
        al, b, w, beta = oracle.gates_from_logits(xa_, a_, **lg_)
        gk = dict(b=b, w=w) if channel else dict(beta=beta)
        o, _ = oracle.fwd(x["q"], x["k"], x["v"], al, h0=x["h0"], nthreads=1, **gk)
        return np.sum(o * dout)

    al, b, w, beta = oracle.gates_from_logits(xa, a_scale, **lg)
    gk = dict(b=b, w=w) if channel else dict(beta=beta)
    g = oracle.bwd(x["q"], x["k"], x["v"], al, h0=x["h0"], dout=dout, **gk)
    if channel:
        lgr = oracle.logit_grads(xa, a_scale, g["dalpha"], x_b=lg["x_b"], db=g["db"], x_w=lg["x_w"], dw=g["dw"])
    else:
        lgr = oracle.logit_grads(xa, a_scale, g["dalpha"], x_beta=lg["x_beta"], dbeta=g["dbeta"])
    h = 1e-6
    checks = [("dalpha", xa, lambda v: loss(v, a_scale, lg)),
              ("dalpha_scale", a_scale, lambda v: loss(xa, v, lg))]
    for name, key in (("db", "x_b"), ("dw", "x_w"), ("dbeta", "x_beta")):
        if key in lg:
            checks.append((name, lg[key], lambda v, key=key: loss(xa, a_scale, {**lg, key: v})))
    for name, base, f in checks:
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            p, m = base.copy(), base.copy()
            p[idx] += h
            m[idx] -= h
            fd[idx] = (f(p) - f(m)) / (2 * h)
        assert relerr(lgr[name], fd) < 1e-6, name


def test_layer_core_forward_closed_forms():
    """The oracle's layer composition (conv k=4 + SiLU, L2 norm of q and k, the recurrence, the
    swish(z) gate; explainer «Architecture et versions hybrides», Figure 1 caption; mkdocs chapter
    «Gated DeltaNet») against closed forms that fix the conv tap orientation, the channel order of
    the convolution weights (q, k, v) and the order of the steps:
    - only the current-token tap, alpha = 1, beta = 0: the state stays h0, so
      y_t = swish(z_t) * h0^T l2(silu(xq_t));
    - only the oldest tap: token t sees xq_{t-3}; the first three tokens see zeros (SiLU(0) = 0,
      and the L2 norm of 0 is 0), so their y is 0;
    - one token, alpha = 1, beta = 1, h0 = 0: S = k v^T, so y = swish(z) * v (k . q) with
      q = l2(silu(xq)), k = l2(silu(2 xk)), v = silu(3 xv) when the current-token tap weighs the
      q, k, v channel blocks 1, 2, 3 (a misplaced block would differ)."""
    rng = np.random.default_rng(41)
    B, T, Hk, Hv, d = 1, 6, 1, 2, 4
    cch = 2 * Hk * d + Hv * d
    xq = rng.standard_normal((B, T, Hk, d))
    xk = rng.standard_normal((B, T, Hk, d))
    xv = rng.standard_normal((B, T, Hv, d))
    z = rng.standard_normal((B, T, Hv, d))
    h0 = rng.standard_normal((B, Hv, d, d))
    silu = lambda x: x / (1.0 + np.exp(-x))
    swish = lambda x: x / (1.0 + np.exp(-x))
    l2 = lambda x: x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + 1e-6)
    ones = np.ones((B, T, Hv))
    zeros = np.zeros((B, T, Hv))
    # current-token tap only
    w = np.zeros((cch, 4))
    w[:, 3] = 1.0
    y, hT = oracle.layer_core_fwd(xq, xk, xv, w, ones, zeros, z, h0=h0)
    q = l2(silu(xq))
    for hv in range(Hv):
        want = swish(z[:, :, hv]) * np.einsum("bij,bti->btj", h0[:, hv], q[:, :, 0])
        np.testing.assert_allclose(y[:, :, hv], want, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(hT, h0, rtol=0, atol=1e-14)
    # oldest tap only: token t reads xq_{t-3}
    w = np.zeros((cch, 4))
    w[:, 0] = 1.0
    y, _ = oracle.layer_core_fwd(xq, xk, xv, w, ones, zeros, z, h0=h0)
    np.testing.assert_allclose(y[:, :3], 0.0, atol=1e-14)
    q3 = l2(silu(xq[:, :T - 3]))
    for hv in range(Hv):
        want = swish(z[:, 3:, hv]) * np.einsum("bij,bti->btj", h0[:, hv], q3[:, :, 0])
        np.testing.assert_allclose(y[:, 3:, hv], want, rtol=1e-12, atol=1e-14)
    # one token, a full write from a zero state; the current tap weighs the q, k and v channel
    # blocks 1, 2 and 3, so a misplaced block changes the result
    cq = Hk * d
    w = np.zeros((cch, 4))
    w[:cq, 3], w[cq:2 * cq, 3], w[2 * cq:, 3] = 1.0, 2.0, 3.0
    y, hT = oracle.layer_core_fwd(xq[:, :1], xk[:, :1], xv[:, :1], w, ones[:, :1], ones[:, :1], z[:, :1])
    qn, kn, vs = l2(silu(xq[:, 0, 0])), l2(silu(2.0 * xk[:, 0, 0])), silu(3.0 * xv[:, 0])
    for hv in range(Hv):
        want = swish(z[:, 0, hv]) * vs[:, hv] * np.sum(kn * qn, axis=-1, keepdims=True)
        np.testing.assert_allclose(y[:, 0, hv], want, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(hT[:, hv], np.einsum("bi,bj->bij", kn, vs[:, hv]), rtol=1e-12, atol=1e-14)
