"""Planted mistakes: each mutant below is a plausible slip in the oracle (a dropped term, a wrong
sign or index, a transposed operand, a wrong tie or threshold rule). The pins in
test_oracle_pins.py must catch every one of them; this test builds each mutant from the oracle's
source on the CPU, points the pins at it and checks that at least one pin fails."""
import inspect
import types

import pytest

from oracle import tt_oracle
import tests.test_oracle_pins as pins

MUTANTS = [
    ("gqa head mapping", "h = kh * G + g", "h = g * Hkv + kh"),
    ("dropped softmax scale", "x = softmax_scale * (q[b, :, h, :] @ keys.T)", "x = (q[b, :, h, :] @ keys.T)"),
    ("keys used as values", "vals = np.concatenate([vs[b][:, kh, :]", "vals = np.concatenate([ks[b][:, kh, :]"),
    ("row max over wrong axis", "m = x.max(axis=1, keepdims=True)", "m = x.max(axis=0, keepdims=True)"),
    ("page table ignored", "p = int(page_table[b][t // page_size])", "p = t // page_size"),
    ("ragged page tail read", "n = min(page_size, L - t)", "n = page_size"),
    ("sin/cos swapped", "np.concatenate([np.cos(arg), np.sin(arg)], axis=1)", "np.concatenate([np.sin(arg), np.cos(arg)], axis=1)"),
    ("frequency exponent", "w = max_period ** (-k / half)", "w = max_period ** (-k / freq_dim)"),
    ("transposed W2", "a2 = silu(a1 @ w2.T + b2)", "a2 = silu(a1 @ w2 + b2)"),
    ("dropped layer embedding", "return out.reshape(-1, 3, D) + emb[None, :, :]", "return out.reshape(-1, 3, D)"),
    ("scale without 1+", "return h / rms * w * (1.0 + scale) + shift", "return h / rms * w * scale + shift"),
    ("sum instead of mean", "np.mean(h * h, axis=-1, keepdims=True)", "np.sum(h * h, axis=-1, keepdims=True)"),
    ("shift/scale rows swapped", "shift = mod[:, 0, :][:, None, :]", "shift = mod[:, 1, :][:, None, :]"),
    ("gate dropped", "return h + gate * f", "return h + f"),
    ("argmax ties to last id", "a = np.argmax(x, axis=-1)", "a = x.shape[-1] - 1 - np.argmax(x[..., ::-1], axis=-1)"),
    ("temperature dropped", "z = np.exp(inv_temperature * (x - m)).sum(axis=-1)", "z = np.exp((x - m)).sum(axis=-1)"),
    ("strict threshold", "chosen = {l for l in masked if conf[b, l] >= gamma}", "chosen = {l for l in masked if conf[b, l] > gamma}"),
    ("position ties to last", "key=lambda l: (-conf[b, l], l)", "key=lambda l: (-conf[b, l], -l)"),
    ("floor schedule", "need = -(-len(masked) // remaining_steps)", "need = len(masked) // remaining_steps"),
    ("tau from committed count", "tau = is_masked.sum(axis=1) / block_size", "tau = (~is_masked).sum(axis=1) / block_size"),
    ("no fallback", "if len(chosen) < need:", "if False:"),
    ("predict-noise ignores exclusion",
     'positions are never changed."""\n    conf, arg = confidence_argmax(logits, inv_temperature, exclude_token)',
     'positions are never changed."""\n    conf, arg = confidence_argmax(logits, inv_temperature)'),
    ("schedule rounds up", "return (block_size * (steps - r)) // steps", "return -(-(block_size * (steps - r)) // steps)"),
]

PIN_TESTS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


def _run_pins():
    failures = 0
    for fn in PIN_TESTS:
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        cases = [()]
        if params:
            names = params[0].args[0]
            single = isinstance(names, str) and "," not in names
            cases = [(c,) for c in params[0].args[1]] if single else params[0].args[1]
        for case in cases:
            try:
                fn(*case)
            except Exception:
                failures += 1
    return failures


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, monkeypatch):
    src = inspect.getsource(tt_oracle)
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    monkeypatch.setattr(pins, "O", mod)
    assert _run_pins() > 0, f"no pin caught the planted mistake: {name}"


def test_unmutated_oracle_passes_all_pins():
    assert _run_pins() == 0
