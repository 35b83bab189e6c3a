"""The oracle pins must catch plausible mistakes.

Each case plants one slip in a private copy of the oracle's source (on the CPU,
never in the CUDA path), swaps the copy in, and checks that at least one pin in
``test_oracle_pins`` fails.
"""
import inspect
import types

import pytest

import oracle
import oracle.zebra as zebra
import tests.test_oracle_pins as pins

MUTATIONS = {
    "bias in log2 units": ("np.log(n[lm].astype(np.float64))", "np.log2(n[lm].astype(np.float64))"),
    "landmark bias dropped": ("+ np.log(n[lm].astype(np.float64))[None, :]", ""),
    "landmark value = mean key": ("value_parts.append(Vbar[h, lm])", "value_parts.append(Kbar[h, lm])"),
    "selected tiles also landmarks": ("mask[sel] = False", "pass"),
    "ties go to the upper index": ("order = np.lexsort((j, -flat[r]))", "order = np.lexsort((-j, -flat[r]))"),
    "softmax scale dropped": ("logit_parts = [scale * q @ K[h, cols].T]", "logit_parts = [q @ K[h, cols].T]"),
    "feature map off by one": ("x + 1.0, np.exp", "x, np.exp"),
    "fit without intercept": ("b[h] = ym - xm @ W", "b[h] = 0.0 * ym"),
    "ridge on the wrong side": ("D = np.concatenate([Xc, np.sqrt(lam) * np.eye(d)], axis=0)",
                                "D = np.concatenate([Xc, -np.sqrt(lam) * np.eye(d) + 1.0], axis=0)"),
    "score transposed": ("np.matmul(Qbar, np.swapaxes(Kbar, -1, -2))",
                         "np.swapaxes(np.matmul(Qbar, np.swapaxes(Kbar, -1, -2)), -1, -2)"),
    "ragged tile divided by full size": ("out /= n[None, :, None].astype(np.float64)", "out /= float(tile)"),
    "keys not centred": ("return linear_state(K - key_mean(K)[..., None, :], V)", "return linear_state(K, V)"),
    "keys centred with the wrong sign": ("linear_state(K - key_mean(K)", "linear_state(K + key_mean(K)"),
    "key mean over the features": ("K.sum(axis=-2) / K.shape[-2]", "K.sum(axis=-1) / K.shape[-1]"),
    "key mean divided by d": ("K.sum(axis=-2) / K.shape[-2]", "K.sum(axis=-2) / K.shape[-1]"),
    "queries centred instead of keys": ("S, z = linear_state_centered(K, V)\n    return linear_apply(Q, S, z, A, b)",
                                        "S, z = linear_state(K, V)\n    return linear_apply(Q - key_mean(Q)[..., None, :], S, z, A, b)"),
    "block mass without the scale": ("P = _softmax_rows(scale * Q[h, r0:r0 + nb[a]] @ K[h].T)",
                                     "P = _softmax_rows(Q[h, r0:r0 + nb[a]] @ K[h].T)"),
    "block mass averaged over rows": ("np.add.reduceat(P.sum(axis=0), starts)", "np.add.reduceat(P.mean(axis=0), starts)"),
    "lightest blocks kept": ("heavy_first = -np.sort(-M, axis=-1)", "heavy_first = np.sort(M, axis=-1)"),
    "selected mass not normalised": ("return kept.sum(axis=-1) / M.sum(axis=-1)", "return kept.sum(axis=-1)"),
}


def _pin_tests():
    return [f for name, f in inspect.getmembers(pins, inspect.isfunction) if name.startswith("test_")]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    old, new = MUTATIONS[name]
    src = inspect.getsource(zebra)
    assert old in src
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    for fn in zebra.__all__:
        monkeypatch.setattr(oracle, fn, getattr(mod, fn))
    failures = 0
    for test in _pin_tests():
        try:
            test()
        except (AssertionError, ValueError, IndexError):
            failures += 1
    assert failures > 0, f"no pin catches: {name}"
