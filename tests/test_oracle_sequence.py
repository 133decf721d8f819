"""Pins of the oracle's layer-by-layer prefill against its token-by-token form.

The layer-major form is only a different loop order of the same causal forward pass:
every position must end with the same logits, DeltaNet states, conv history and KV
cache as ``oracle.prefill``, which feeds the prompt one decode step at a time. These
checks run on small models, fresh and continued states, both DeltaNet evaluations
(the recurrence and its chunked form), the bf16-activation diagnostic and the 8-bit
KV cache.
"""
import numpy as np
import pytest

import oracle
import synth


def _weights(cfg):
    return oracle.prepare_weights(cfg, synth.make_weights(cfg))


@pytest.fixture(scope="module")
def tiny():
    cfg = synth.TINY
    return cfg, _weights(cfg)


@pytest.fixture(scope="module")
def mini():
    cfg = synth.MINI
    return cfg, _weights(cfg)


def _same_state(cfg, a, b, tol):
    assert a.pos == b.pos
    for x, y in zip(a.S, b.S):
        assert np.abs(x - y).max() <= tol * max(1.0, np.abs(y).max())
    for x, y in zip(a.conv, b.conv):
        assert np.abs(x - y).max() <= tol * max(1.0, np.abs(y).max())
    for x, y in zip(a.K + a.V, b.K + b.V):
        # bf16 entries: float64 addition order may move a value across a rounding midpoint
        # only when it lies within ~1e-15 of one; the entries must then differ by one ulp
        d = np.abs(x - y)
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(y), 1e-30))) - 7)
        assert np.all(d <= ulp), float(np.max(d / ulp))
        assert (d > 0).mean() < 1e-3


@pytest.mark.parametrize("chunk", [None, 7, 64])
def test_sequence_equals_token_by_token(tiny, chunk):
    cfg, W = tiny
    prompt = synth.make_prompt(cfg, 70, tag="seq")
    a = oracle.new_state(cfg, 160)
    b = oracle.new_state(cfg, 160)
    za = oracle.prefill_sequence(cfg, W, a, prompt, chunk=chunk)
    zb = oracle.prefill(cfg, W, b, prompt)
    assert np.abs(za - zb).max() <= 1e-9 * max(1.0, np.abs(zb).max())
    _same_state(cfg, a, b, 1e-9)


def test_sequence_continues_from_state(tiny):
    cfg, W = tiny
    p1 = synth.make_prompt(cfg, 23, tag="seq-a")
    p2 = synth.make_prompt(cfg, 41, tag="seq-b")
    a = oracle.new_state(cfg, 160)
    b = oracle.new_state(cfg, 160)
    oracle.prefill_sequence(cfg, W, a, p1)
    oracle.prefill(cfg, W, b, p1)
    za = oracle.prefill_sequence(cfg, W, a, p2, chunk=16)
    zb = oracle.prefill(cfg, W, b, p2)
    assert np.abs(za - zb).max() <= 1e-9 * max(1.0, np.abs(zb).max())
    _same_state(cfg, a, b, 1e-9)


def test_sequence_single_token_is_a_decode_step(mini):
    cfg, W = mini
    a = oracle.new_state(cfg, 16)
    b = oracle.new_state(cfg, 16)
    za = oracle.prefill_sequence(cfg, W, a, np.array([5]))
    zb = oracle.decode_step(cfg, W, b, 5)
    assert np.abs(za - zb).max() <= 1e-12
    _same_state(cfg, a, b, 1e-12)


def test_sequence_bf16_activations(mini):
    cfg, W = mini
    prompt = synth.make_prompt(cfg, 33, tag="seq-act")
    a = oracle.new_state(cfg, 40)
    b = oracle.new_state(cfg, 40)
    za = oracle.prefill_sequence(cfg, W, a, prompt, act_bf16=True)
    zb = oracle.prefill(cfg, W, b, prompt, act_bf16=True)
    assert np.abs(za - zb).max() <= 1e-9 * max(1.0, np.abs(zb).max())
    for x, y in zip(a.S, b.S):
        assert np.abs(x - y).max() <= 1e-9


def test_sequence_q8_cache(tiny):
    cfg, W = tiny
    prompt = synth.make_prompt(cfg, 45, tag="seq-q8")
    a = oracle.new_state(cfg, 64, kv_q8=True)
    b = oracle.new_state(cfg, 64, kv_q8=True)
    za = oracle.prefill_sequence(cfg, W, a, prompt, chunk=16)
    zb = oracle.prefill(cfg, W, b, prompt)
    assert np.abs(za - zb).max() <= 1e-9 * max(1.0, np.abs(zb).max())
    for x, y in zip(a.K + a.V, b.K + b.V):
        assert (np.abs(x - y) > 1e-12).mean() < 1e-3


def test_sequence_causal_attention_brute_force():
    """Each query row equals the single-query decode attention over its own prefix."""
    rng = np.random.default_rng(3)
    T, Hq, Hkv, D, pos0 = 9, 4, 2, 8, 5
    q = rng.standard_normal((T, Hq, D))
    K = rng.standard_normal((Hkv, pos0 + T + 3, D))
    V = rng.standard_normal((Hkv, pos0 + T + 3, D))
    got = oracle.causal_attention(q, K, V, pos0)
    for t in range(T):
        n = pos0 + t + 1
        want = oracle.attention_decode(q[t], K[:, :n], V[:, :n])
        assert np.abs(got[t] - want).max() <= 1e-12


def test_sequence_rope_positions_matches_scalar_rope():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((6, 3, 16))
    pos = np.array([0, 1, 7, 100, 4095, 32767])
    got = oracle.rope_positions(x, pos, 1e7)
    for t in range(6):
        assert np.abs(got[t] - oracle.rope(x[t], int(pos[t]), 1e7)).max() <= 1e-12


def test_sequence_planted_slip_is_caught(tiny):
    """A slip in the layer-major loop (conv window not carried) must break the equality."""
    cfg, W = tiny
    p1 = synth.make_prompt(cfg, 12, tag="slip-a")
    p2 = synth.make_prompt(cfg, 12, tag="slip-b")
    a = oracle.new_state(cfg, 64)
    b = oracle.new_state(cfg, 64)
    oracle.prefill_sequence(cfg, W, a, p1)
    oracle.prefill(cfg, W, b, p1)
    for li in range(cfg.n_dn):
        a.conv[li] = np.zeros_like(a.conv[li])
    za = oracle.prefill_sequence(cfg, W, a, p2)
    zb = oracle.prefill(cfg, W, b, p2)
    assert np.abs(za - zb).max() > 1e-6
