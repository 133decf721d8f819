"""Pins for the oracle's sampling-mode speculative verify.

What fixes it, independently of its own code:
  * softmax with temperature: the two-token closed form (a logistic function);
  * the inverse-CDF draw: brute force over a lattice of uniforms reproduces the
    weights' proportions, and never picks a zero-weight token;
  * distribution preservation (the property the follow-up post claims): over a
    lattice of both uniforms, the first emitted token is distributed exactly as the
    target p, whatever the draft; for two drafts, the joint law of the emitted
    prefix is p_0(x_1) p_1(x_2) ... (seeded Monte Carlo within 5 sigma);
  * temperature -> 0 is the greedy rule (longest prefix of drafts equal to the
    argmax, then the argmax), checked against that rule written out here and against
    the oracle's greedy verify on the tiny model.
"""
import math

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_softmax_t_two_token_closed_form():
    for z0, z1, tau in [(0.3, -1.2, 1.0), (2.0, 2.5, 0.25), (-4.0, 3.0, 7.0)]:
        p = oracle.softmax_t(np.array([z0, z1]), tau)
        p0 = 1.0 / (1.0 + math.exp((z1 - z0) / tau))
        assert abs(p[0] - p0) < 1e-15 and abs(p[1] - (1.0 - p0)) < 1e-15


def test_softmax_t_rejects_nonpositive_temperature():
    with pytest.raises(ValueError):
        oracle.softmax_t(np.zeros(3), 0.0)


def test_inverse_cdf_lattice_proportions():
    w = np.array([0.0, 3.0, 1.0, 0.0, 0.5, 2.5, 0.0])
    N = 20000
    counts = np.zeros(w.size)
    for k in range(N):
        j, _ = oracle.inverse_cdf(w, (k + 0.5) / N)
        counts[j] += 1
    assert counts[w == 0].sum() == 0
    np.testing.assert_allclose(counts / N, w / w.sum(), atol=1.0 / N)


def test_inverse_cdf_edges():
    w = np.array([0.0, 0.0, 1.0, 1.0])
    assert oracle.inverse_cdf(w, 0.0)[0] == 2          # r = 0: the first token with weight
    assert oracle.inverse_cdf(w, 0.5)[0] == 3          # exactly on a boundary: the next token
    assert oracle.inverse_cdf(w, np.nextafter(1.0, 0))[0] == 3
    assert oracle.inverse_cdf(np.array([0.0, 5.0, 0.0]), 0.9)[0] == 1


def _brute_first_token_law(logits_row, draft, tau, N):
    """Law of the first emitted token over an N x N lattice of (u, r), K = 1."""
    V = logits_row.size
    counts = np.zeros(V)
    logits = np.stack([logits_row, logits_row])       # row 1 only matters when the draft is kept
    for a in range(N):
        for b in range(N):
            u = np.array([[(a + 0.5) / N, (b + 0.5) / N], [0.5, 0.5]])
            _, out, _ = oracle.accept_sampled(logits, [draft], tau, u)
            counts[out[0]] += 1
    return counts / (N * N)


@pytest.mark.parametrize("draft", [0, 2, 4])
def test_first_token_law_equals_target(draft):
    z = np.array([0.7, -0.4, 1.1, 0.0, -1.5])
    tau = 0.8
    p = oracle.softmax_t(z, tau)
    law = _brute_first_token_law(z, draft, tau, 160)
    np.testing.assert_allclose(law, p, atol=3.0 / 160)


def test_joint_law_two_drafts_monte_carlo():
    rng = np.random.default_rng(7)
    V, tau = 5, 0.9
    logits = rng.standard_normal((3, V)) * 1.3
    d1, d2 = int(np.argmax(logits[0])), int(np.argsort(logits[1])[-2])
    p = [oracle.softmax_t(logits[i], tau) for i in range(3)]
    M = 20000
    n_hist = np.zeros(3)
    first = np.zeros(V)
    second = np.zeros(V)      # out[1] given out[0] == d1
    third = np.zeros(V)       # out[2] given out[:2] == [d1, d2]
    for _ in range(M):
        n, out, _ = oracle.accept_sampled(logits, [d1, d2], tau, rng.random((3, 2)))
        n_hist[n] += 1
        first[out[0]] += 1
        if out[0] == d1 and len(out) > 1:
            second[out[1]] += 1
            if out[1] == d2 and len(out) > 2:
                third[out[2]] += 1
    tol = 5.0 * math.sqrt(0.25 / M)
    np.testing.assert_allclose(first / M, p[0], atol=tol)
    np.testing.assert_allclose(second / M, p[0][d1] * p[1], atol=tol)
    np.testing.assert_allclose(third / M, p[0][d1] * p[1][d2] * p[2], atol=tol)
    # acceptance counts: P(n >= 1) = p_0(d1), P(n = 2) = p_0(d1) p_1(d2)
    assert abs((n_hist[1] + n_hist[2]) / M - p[0][d1]) < tol
    assert abs(n_hist[2] / M - p[0][d1] * p[1][d2]) < tol


def _greedy_rule(logits, drafts):
    g = [int(np.argmax(r)) for r in logits]
    n = 0
    while n < len(drafts) and drafts[n] == g[n]:
        n += 1
    return n, list(drafts[:n]) + [g[n]]


def test_zero_temperature_limit_is_greedy():
    rng = np.random.default_rng(11)
    for trial in range(200):
        K, V = 4, 50
        logits = rng.permutation(V * (K + 1)).reshape(K + 1, V) * 0.01   # distinct values, gaps >= 0.01
        g = [int(np.argmax(r)) for r in logits]
        drafts = [g[i] if rng.random() < 0.7 else int(rng.integers(V)) for i in range(K)]
        n, out, _ = oracle.accept_sampled(logits, drafts, 1e-4, rng.random((K + 1, 2)))
        n_ref, out_ref = _greedy_rule(logits, drafts)
        assert n == n_ref and list(out) == out_ref, trial


def test_rejected_draft_is_never_emitted_at_its_position():
    rng = np.random.default_rng(3)
    z = np.array([3.0, 0.0, 0.0])
    for _ in range(500):
        n, out, _ = oracle.accept_sampled(np.stack([z, z]), [0], 1.0, rng.random((2, 2)))
        if n == 0:
            assert out[0] != 0


def test_model_level_sampled_verify_at_zero_temperature_equals_greedy_verify():
    cfg = synth.TINY
    W = oracle.prepare_weights(cfg, synth.make_weights(cfg))
    prompt = synth.make_prompt(cfg, 12, seed=5)
    st = oracle.new_state(cfg, 64)
    z = oracle.prefill(cfg, W, st, prompt)
    last = int(np.argmax(z))
    greedy, _ = oracle.greedy_generate(cfg, W, st.copy(), last, 3)
    drafts = [int(greedy[0]), int(greedy[1]), (int(greedy[2]) + 1) % cfg.vocab]
    st_g, st_s = st.copy(), st.copy()
    n_g, out_g, logits_g = oracle.verify_drafts(cfg, W, st_g, last, drafts)
    u = np.random.default_rng(0).random((4, 2))
    n_s, out_s, logits_s, _ = oracle.verify_drafts_sampled(cfg, W, st_s, last, drafts, 1e-6, u)
    assert n_g == n_s == 2
    assert list(out_g) == list(out_s)
    np.testing.assert_array_equal(logits_g, logits_s)
    assert st_s.pos == st_g.pos
    for a, b in zip(st_s.S, st_g.S):
        np.testing.assert_array_equal(a, b)


# ------------------------------------------------------------------ planted mistakes (CPU only)
def _accept_keeps_draft_in_residual(logits, drafts, tau, uniforms):
    p = oracle.softmax_t(logits[0], tau)
    if uniforms[0, 0] < p[drafts[0]]:
        return 1, np.array([drafts[0], 0], dtype=np.int32), 1.0
    tok, _ = oracle.inverse_cdf(p, uniforms[0, 1])       # slip: the rejected draft stays in
    return 0, np.array([tok], dtype=np.int32), 1.0


def _accept_inverted_test(logits, drafts, tau, uniforms):
    p = oracle.softmax_t(logits[0], tau)
    if uniforms[0, 0] > p[drafts[0]]:                      # slip: keeps with probability 1 - p(d)
        return 1, np.array([drafts[0], 0], dtype=np.int32), 1.0
    resid = p.copy()
    resid[drafts[0]] = 0.0
    tok, _ = oracle.inverse_cdf(resid, uniforms[0, 1])
    return 0, np.array([tok], dtype=np.int32), 1.0


def _softmax_times_tau(z, tau):
    x = np.asarray(z, dtype=np.float64) * tau              # slip: multiplies by the temperature
    w = np.exp(x - x.max())
    return w / w.sum()


@pytest.mark.parametrize("name,fn", [
    ("accept_sampled", _accept_keeps_draft_in_residual),
    ("accept_sampled", _accept_inverted_test),
    ("softmax_t", _softmax_times_tau),
])
def test_planted_sampling_mistake_is_caught(monkeypatch, name, fn):
    monkeypatch.setattr(oracle, name, fn)
    import oracle.sampling as osm
    monkeypatch.setattr(osm, name, fn)
    z = np.array([0.7, -0.4, 1.1, 0.0, -1.5])
    tau = 0.8
    p = np.exp(z / tau) / np.exp(z / tau).sum()            # the target, written out independently
    law = _brute_first_token_law(z, 0, tau, 60)             # p(draft) = 0.30, far from 1/2
    assert np.max(np.abs(law - p)) > 0.05
