"""Planted mistakes in the oracle (on the CPU only) must be caught by the pins.

Each case patches one oracle function with a plausible slip and checks that the
independent plain-Python model then disagrees with the oracle.
"""
import numpy as np
import pytest

import oracle
import oracle.model as om
import synth
from pyref_model import PyModel

MINI = synth.MINI


def _max_diff(W, raw):
    py = PyModel(MINI, raw)
    st = oracle.new_state(MINI, 32)
    worst = 0.0
    for t in [5, 9, 33, 2, 50]:
        z1 = oracle.decode_step(MINI, W, st, t)
        z2 = np.array(py.step(t))
        worst = max(worst, float(np.max(np.abs(z1 - z2))))
    return worst


def _no_decay_in_correction(S, q, k, v, a, b):          # uses S instead of a*S in S k
    Sd = a * S
    S_new = Sd - b * np.outer(S @ k, k) + b * np.outer(v, k)
    return S_new, S_new @ q


def _readout_before_update(S, q, k, v, a, b):
    Sd = a * S
    S_new = Sd - b * np.outer(Sd @ k, k) + b * np.outer(v, k)
    return S_new, S @ q


def _rope_wrong_sign(x, pos, theta):
    D = x.shape[-1]
    half = D // 2
    ang = pos * theta ** (-2.0 * np.arange(half) / D)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * np.cos(ang) + x2 * np.sin(ang), x1 * np.sin(ang) + x2 * np.cos(ang)], axis=-1)


def _rmsnorm_no_gain(h, gamma, eps):
    return h / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps)


def _conv_tap_reversed(window, x_t, taps):
    full = np.concatenate([window, x_t[None, :]], axis=0)
    return om.silu(np.einsum("wc,cw->c", full[::-1], taps))


@pytest.mark.parametrize("name,fn", [
    ("delta_rule_step", _no_decay_in_correction),
    ("delta_rule_step", _readout_before_update),
    ("rope", _rope_wrong_sign),
    ("rmsnorm", _rmsnorm_no_gain),
    ("conv_silu", _conv_tap_reversed),
])
def test_planted_mistake_is_caught(monkeypatch, name, fn):
    raw = synth.make_weights(MINI)
    W = oracle.prepare_weights(MINI, raw)
    assert _max_diff(W, raw) < 1e-9                  # the unpatched oracle agrees
    monkeypatch.setattr(om, name, fn)
    assert _max_diff(W, raw) > 1e-6                  # the slip shows up


def test_planted_chunk_mask_mistake_is_caught(monkeypatch):
    import oracle.chunked as oc
    r = np.random.default_rng(0)
    T, dk, dv = 20, 6, 5
    Q = oracle.l2norm(r.standard_normal((T, dk)))
    K = oracle.l2norm(r.standard_normal((T, dk)))
    V = r.standard_normal((T, dv))
    a = np.full(T, 0.6)
    b = np.full(T, 0.5)
    S0 = r.standard_normal((dv, dk))
    O1, _ = oracle.deltanet_recurrent(S0, Q, K, V, a, b)
    real_tril = np.tril

    def off_by_one_tril(m, k=0):                      # drops the diagonal from the output mask
        return real_tril(m, k=-1)

    monkeypatch.setattr(oc.np, "tril", off_by_one_tril)
    O2, _ = oc.deltanet_chunked(S0, Q, K, V, a, b, 7)
    monkeypatch.setattr(oc.np, "tril", real_tril)
    assert np.max(np.abs(O2 - O1)) > 1e-3
