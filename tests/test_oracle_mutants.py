"""The pins must bite: plausible mistakes planted in a copy of the oracle (the compiled recurrence,
and the numpy reverse mode of the layer core) each make at least one pin of test_oracle_pins.py
fail."""
import os
import shutil
import subprocess
import tempfile

import pytest

from oracle import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.cpp")

# (name, [(original text, planted mistake)])
MUTANTS = [
    ("erase along the gated key e instead of k",
     [("S[i * dv + j] += x.k[i] * u[j];", "S[i * dv + j] += e[i] * u[j];")]),
    ("read the old value with k instead of e",
     [("u[j] -= e[i] * S[i * dv + j];", "u[j] -= x.k[i] * S[i * dv + j];")]),
    ("decay applied after the write instead of before",
     [("for (int j = 0; j < dv; ++j) S[i * dv + j] *= ai;", "(void)ai;"),
      ("S[i * dv + j] += x.k[i] * u[j];",
       "S[i * dv + j] = (S[i * dv + j] + x.k[i] * u[j]) * x.a[d.a_ch == 1 ? 0 : i];")]),
    ("readout scale dropped", [("o[j] *= scale;", "o[j] *= 1.0;")]),
    ("write gate indexed by the wrong channel",
     [("u[j] = x.wg[d.w_ch == 1 ? 0 : j] * x.v[j];", "u[j] = x.wg[0] * x.v[j];")]),
    ("channel decay collapsed to its first channel",
     [("double ai = x.a[d.a_ch == 1 ? 0 : i];\n        for (int j = 0; j < dv; ++j) S[i * dv + j] *= ai;",
       "double ai = x.a[0];\n        for (int j = 0; j < dv; ++j) S[i * dv + j] *= ai;")]),
    ("GQA map ignored", [("int hk = map[hv];", "int hk = hv % d.Hk;")]),
    ("backward: sign of the erase-gradient flipped", [("de[i] = -acc;", "de[i] = acc;")]),
    ("backward: decay dropped when passing dS to the previous step",
     [("for (int j = 0; j < dv; ++j) dS[i * dv + j] = ai * dSbar[i * dv + j];",
       "for (int j = 0; j < dv; ++j) dS[i * dv + j] = dSbar[i * dv + j]; (void)ai;")]),
    ("backward: readout term added after dk is taken",
     [("for (int j = 0; j < dv; ++j) dS[i * dv + j] += scale * x.q[i] * gout[j];",
       "for (int j = 0; j < dv; ++j) dS[i * dv + j] += 0.0 * x.q[i] * gout[j];")]),
    ("chunk form: decay ratio inverted",
     [("double ratio = std::exp(g[r * dk + c] - g[s * dk + c]);",
       "double ratio = std::exp(g[s * dk + c] - g[r * dk + c]);")]),
    ("chunk form: triangular solve sign flipped",
     [("acc -= A[r * C + s] * Tm[s * C + col];", "acc += A[r * C + s] * Tm[s * C + col];")]),
    ("conv taps reversed", [("acc += w[ch * 4 + i] * in(t - 3 + i);", "acc += w[ch * 4 + 3 - i] * in(t - 3 + i);")]),
]


def _run_pins():
    """Run every pin; return the names of those that fail."""
    calls = [
        ("worked example", pins.test_worked_example_three_rules, ()),
        ("gdn reduction", pins.test_reduction_to_gated_deltanet, ()),
        ("deltanet reduction", pins.test_reduction_to_deltanet, ()),
        ("linear closed form", pins.test_linear_attention_closed_form, ()),
        ("decay closed form", pins.test_decay_only_closed_form, ()),
        ("exact recall", pins.test_exact_recall_unit_key, ()),
        ("edit invariant", pins.test_edit_invariant, ()),
        ("orthogonal spare", pins.test_orthogonal_keys_spared, ()),
        ("gqa", pins.test_gqa_equals_replicated_heads, ()),
        ("chunk form channel", pins.test_chunk_form_matches_sequential, (16, True)),
        ("chunk form scalar", pins.test_chunk_form_matches_sequential, (16, False)),
        ("bwd fd gdn2", pins.test_backward_finite_differences, ("gdn2",)),
        ("bwd fd gdn", pins.test_backward_finite_differences, ("gdn",)),
        ("conv", pins.test_conv_matches_library_convolution_and_carries_history, ()),
    ]
    failed = []
    for name, fn, args in calls:
        try:
            fn(*args)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(name)
    return failed


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def test_unmutated_oracle_passes_every_pin():
    assert _run_pins() == []


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, edits, workdir):
    src = open(SRC).read()
    for old, new in edits:
        assert old in src, f"mutation anchor not found: {old!r}"
        src = src.replace(old, new)
    tag = str(abs(hash(name)))
    cpp = os.path.join(workdir, f"m{tag}.cpp")
    so = os.path.join(workdir, f"m{tag}.so")
    with open(cpp, "w") as f:
        f.write(src)
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-fPIC", "-shared", "-pthread", cpp, "-o", so])
    saved = oracle._load()
    oracle._lib = oracle.load_library(so)
    try:
        failed = _run_pins()
    finally:
        oracle._lib = saved
    assert failed, f"no pin caught the planted mistake: {name}"


# The layer core's reverse mode is numpy code in oracle.py: (name, original text, planted mistake).
# Each lives in the backward only (the layer pin's forward runs through the compiled conv and
# recurrence), so the finite-difference pin must catch it.
PY = os.path.join(os.path.dirname(oracle.__file__), "oracle.py")
LAYER_MUTANTS = [
    ("swish gate: dz without its z s (1 - s) term",
     "dswz = sg + zz * sg * (1.0 - sg)", "dswz = sg"),
    ("swish gate: do without the factor z", "swz = zz * sg ", "swz = sg "),
    ("output norm backward without the mean term",
     "do = r * (dn - n * np.mean(dn * n, axis=-1, keepdims=True))", "do = r * dn"),
    ("output norm: weight gradient without the gate",
     'extra["dnorm_w"] = np.sum(g * n * swz, axis=(0, 1, 2))', 'extra["dnorm_w"] = np.sum(g * n, axis=(0, 1, 2))'),
    ("output norm: dz without the norm weight", "dz = g * n * wn * dswz", "dz = g * n * dswz"),
    ("L2 norm backward without the projection",
     "da = ((gout - out * dot) / n).reshape(a.shape)", "da = (gout / n).reshape(a.shape)"),
    ("SiLU backward: the sigmoid's derivative instead of SiLU's",
     "du = da * (s + u * s * (1.0 - s))", "du = da * s * (1.0 - s)"),
    ("conv input gradient: taps reversed",
     "dx[:, :T - sh] += w[:, tap] * du[:, sh:]", "dx[:, :T - sh] += w[:, 3 - tap] * du[:, sh:]"),
    ("conv weight gradient: current tap shifted by one token",
     "dw[:, tap] = np.sum(du * x, axis=(0, 1))", "dw[:, tap] = np.sum(du[:, 1:] * x[:, :-1], axis=(0, 1))"),
    ("recomputed conv: history taps shifted the wrong way",
     "u[:, sh:] += w[:, tap] * x[:, :T - sh]", "u[:, :T - sh] += w[:, tap] * x[:, sh:]"),
]


def _oracle_copy(src):
    import types
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = oracle.__file__
    exec(compile(src, PY, "exec"), mod.__dict__)
    return mod


def _layer_pins():
    """The finite-difference pins of the layer core's reverse mode, with and without the output norm."""
    return [lambda: pins.test_layer_backward_finite_differences(False),
            lambda: pins.test_layer_backward_finite_differences(True),
            pins.test_layer_backward_with_output_norm_finite_differences]


def test_unmutated_layer_oracle_copy_passes_its_pin(monkeypatch):
    monkeypatch.setattr(pins, "oracle", _oracle_copy(open(PY).read()))
    for pin in _layer_pins():
        pin()


@pytest.mark.parametrize("name,old,new", LAYER_MUTANTS, ids=[m[0] for m in LAYER_MUTANTS])
def test_planted_layer_backward_mistake_is_caught(name, old, new, monkeypatch):
    src = open(PY).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    monkeypatch.setattr(pins, "oracle", _oracle_copy(src.replace(old, new)))
    caught = []
    for i, pin in enumerate(_layer_pins()):
        try:
            pin()
        except AssertionError:
            caught.append(i)
    assert caught, f"no pin caught the planted mistake: {name}"


# The layer core's forward composition (numpy in oracle.py around the compiled pieces): planted
# mistakes that the closed forms of test_layer_core_forward_closed_forms must catch.
LAYER_FWD_MUTANTS = [
    ("layer forward: q and k convolution weight blocks swapped",
     [("q, _ = conv_silu(xq.reshape(B, T, cq), w[:cq])", "q, _ = conv_silu(xq.reshape(B, T, cq), w[cq:2 * cq])"),
      ("k, _ = conv_silu(xk.reshape(B, T, cq), w[cq:2 * cq])", "k, _ = conv_silu(xk.reshape(B, T, cq), w[:cq])")]),
    ("layer forward: k left without its L2 norm",
     [("k = l2norm(k.reshape(B, T, Hk, dk))", "k = k.reshape(B, T, Hk, dk)")]),
    ("layer forward: v taken before its convolution",
     [("v = v.reshape(B, T, Hv, dv)", "v = xv")]),
]


def test_unmutated_layer_forward_copy_passes_its_pin(monkeypatch):
    monkeypatch.setattr(pins, "oracle", _oracle_copy(open(PY).read()))
    pins.test_layer_core_forward_closed_forms()


@pytest.mark.parametrize("name,edits", LAYER_FWD_MUTANTS, ids=[m[0] for m in LAYER_FWD_MUTANTS])
def test_planted_layer_forward_mistake_is_caught(name, edits, monkeypatch):
    src = open(PY).read()
    for old, new in edits:
        assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
        src = src.replace(old, new)
    monkeypatch.setattr(pins, "oracle", _oracle_copy(src))
    with pytest.raises(AssertionError):
        pins.test_layer_core_forward_closed_forms()
