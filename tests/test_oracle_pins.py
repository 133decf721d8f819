"""Pins for the CPU oracle: each oracle function is checked against something other
than itself (brute force with scalar loops, closed forms, invariants, a library
routine), so that a dropped term, wrong sign, index or transposed operand fails.
"""
import math
import struct

import numpy as np
import pytest
import torch

import oracle
import synth

rng = np.random.default_rng(1234)


# ------------------------------------------------------------------ bf16 rounding
def test_round_bf16_matches_torch():
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 1, 1e3)])
    ours = oracle.round_bf16(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_round_bf16_ties_to_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to the even significand (1.0)
    assert oracle.round_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    # 1 + 3*2^-8 is halfway between 1+2^-7 and 1+2^-6: even is 1+2^-6
    assert oracle.round_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6
    assert oracle.round_bf16(np.array([-(1 + 2 ** -8)]))[0] == -1.0


def test_decode_bf16_bits_known_patterns():
    bits = np.array([0x3F80, 0xBF80, 0x4000, 0x0000, 0x3E80], dtype=np.uint16)
    np.testing.assert_array_equal(oracle.decode_bf16_bits(bits), [1.0, -1.0, 2.0, 0.0, 0.25])


# ------------------------------------------------------------------ elementwise pieces
def test_rmsnorm_brute_force():
    for n in (1, 3, 17):
        h = rng.standard_normal(n) * 3
        g = 1 + rng.standard_normal(n) * 0.1
        ms = sum(v * v for v in h) / n
        ref = [h[i] / math.sqrt(ms + 1e-6) * g[i] for i in range(n)]
        np.testing.assert_allclose(oracle.rmsnorm(h, g, 1e-6), ref, rtol=1e-13)


def test_rmsnorm_unit_rms_property():
    h = rng.standard_normal(1024) * 7
    x = oracle.rmsnorm(h, np.ones(1024), 0.0)
    assert abs(np.sqrt(np.mean(x * x)) - 1) < 1e-12


def test_softplus_and_gates():
    x = np.array([-800.0, -30, -1, 0, 1e-9, 2.5, 30, 800])
    sp = oracle.softplus(x)
    ref = [math.log1p(math.exp(v)) if v < 700 else v for v in x]
    np.testing.assert_allclose(sp, ref, rtol=1e-14, atol=0)
    # exp(-softplus(x)) == sigmoid(-x)
    np.testing.assert_allclose(np.exp(-sp), [1 / (1 + math.exp(v)) if v < 700 else 0.0 for v in x],
                               rtol=1e-12, atol=1e-300)
    assert oracle.sigmoid(np.array([0.0]))[0] == 0.5
    np.testing.assert_allclose(oracle.silu(np.array([1.0])), [1 / (1 + math.exp(-1))])


def test_l2norm_brute_force():
    x = rng.standard_normal((3, 5))
    y = oracle.l2norm(x, 1e-6)
    for r in range(3):
        nrm = math.sqrt(sum(v * v for v in x[r]) + 1e-6)
        np.testing.assert_allclose(y[r], [v / nrm for v in x[r]], rtol=1e-14)


def test_conv_brute_force_and_zero_history():
    C, W = 5, 4
    taps = rng.standard_normal((C, W))
    hist = [rng.standard_normal(C) for _ in range(6)]
    window = np.zeros((W - 1, C))
    for t, x in enumerate(hist):
        y = oracle.conv_silu(window, x, taps)
        for c in range(C):
            acc = 0.0
            for j in range(W):
                src = t - (W - 1) + j
                if src >= 0:
                    acc += taps[c, j] * hist[src][c]
            assert abs(y[c] - acc / (1 + math.exp(-acc))) < 1e-13
        window = np.concatenate([window[1:], x[None]], axis=0)


# ------------------------------------------------------------------ delta rule
def _unit(v):
    return v / np.linalg.norm(v)


def test_delta_rule_b0_only_decays():
    S = rng.standard_normal((6, 4))
    q, k, v = rng.standard_normal(4), _unit(rng.standard_normal(4)), rng.standard_normal(6)
    S1, o = oracle.delta_rule_step(S, q, k, v, 0.37, 0.0)
    np.testing.assert_allclose(S1, 0.37 * S, rtol=1e-15)
    np.testing.assert_allclose(o, 0.37 * S @ q, rtol=1e-14)


def test_delta_rule_a1_b1_unit_k_writes_v():
    S = rng.standard_normal((6, 4))
    k = _unit(rng.standard_normal(4))
    v = rng.standard_normal(6)
    S1, _ = oracle.delta_rule_step(S, rng.standard_normal(4), k, v, 1.0, 1.0)
    np.testing.assert_allclose(S1 @ k, v, rtol=1e-13, atol=1e-13)


def test_delta_rule_orthonormal_keys_closed_form():
    d = 8
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    ks = Qm.T                                   # orthonormal rows
    vs = rng.standard_normal((d, 5))
    S = np.zeros((5, d))
    for i in range(d):
        S, _ = oracle.delta_rule_step(S, ks[i], ks[i], vs[i], 1.0, 1.0)
    np.testing.assert_allclose(S, sum(np.outer(vs[i], ks[i]) for i in range(d)), atol=1e-12)


def test_delta_rule_a1_b0_constant():
    S = rng.standard_normal((3, 3))
    S1, _ = oracle.delta_rule_step(S, *rng.standard_normal((3, 3)), 1.0, 0.0)
    np.testing.assert_array_equal(S1, S)


def test_delta_rule_matches_scalar_loop():
    dv, dk = 3, 4
    S = rng.standard_normal((dv, dk))
    q, k, v = rng.standard_normal(dk), rng.standard_normal(dk), rng.standard_normal(dv)
    a, b = 0.8, 0.3
    S1, o = oracle.delta_rule_step(S, q, k, v, a, b)
    ref = [[0.0] * dk for _ in range(dv)]
    for i in range(dv):
        u = sum(a * S[i][j] * k[j] for j in range(dk))
        for j in range(dk):
            ref[i][j] = a * S[i][j] + b * (v[i] - u) * k[j]
    np.testing.assert_allclose(S1, ref, rtol=1e-13)
    np.testing.assert_allclose(o, [sum(ref[i][j] * q[j] for j in range(dk)) for i in range(dv)], rtol=1e-13)


# ------------------------------------------------------------------ chunked == recurrent
def _dn_inputs(T, dk, dv, seed):
    r = np.random.default_rng(seed)
    Q = oracle.l2norm(r.standard_normal((T, dk)))
    K = oracle.l2norm(r.standard_normal((T, dk)))
    V = r.standard_normal((T, dv))
    a = np.exp(-oracle.softplus(r.standard_normal(T)))       # typical 0.3 .. 0.75
    b = oracle.sigmoid(r.standard_normal(T))
    S0 = r.standard_normal((dv, dk)) * 0.1
    return S0, Q, K, V, a, b


@pytest.mark.parametrize("chunk,T", [(1, 9), (7, 30), (64, 150), (64, 64)])
def test_chunked_equals_recurrent(chunk, T):
    S0, Q, K, V, a, b = _dn_inputs(T, 16, 12, chunk * 100 + T)
    O1, S1 = oracle.deltanet_recurrent(S0, Q, K, V, a, b)
    O2, S2 = oracle.deltanet_chunked(S0, Q, K, V, a, b, chunk)
    np.testing.assert_allclose(O2, O1, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(S2, S1, rtol=1e-9, atol=1e-11)


def test_chunked_strong_decay_is_stable():
    S0, Q, K, V, a, b = _dn_inputs(128, 8, 8, 5)
    a = np.full(128, 0.3)                      # cumulative decay e^{-77} inside a chunk
    O1, S1 = oracle.deltanet_recurrent(S0, Q, K, V, a, b)
    O2, S2 = oracle.deltanet_chunked(S0, Q, K, V, a, b, 64)
    assert np.all(np.isfinite(O2))
    np.testing.assert_allclose(O2, O1, rtol=1e-9, atol=1e-12)


def test_recurrent_reference_matches_step_function():
    S0, Q, K, V, a, b = _dn_inputs(10, 6, 5, 9)
    O1, S1 = oracle.deltanet_recurrent(S0, Q, K, V, a, b)
    S = S0.copy()
    for t in range(10):
        S, o = oracle.delta_rule_step(S, Q[t], K[t], V[t], a[t], b[t])
        np.testing.assert_allclose(o, O1[t], rtol=1e-12)
    np.testing.assert_allclose(S, S1, rtol=1e-12)


# ------------------------------------------------------------------ RoPE and attention
def test_rope_properties():
    D = 16
    q, k = rng.standard_normal(D), rng.standard_normal(D)
    np.testing.assert_array_equal(oracle.rope(q, 0, 1e7), q)
    for p in (1, 5, 1000, 32767):
        assert abs(np.linalg.norm(oracle.rope(q, p, 1e7)) - np.linalg.norm(q)) < 1e-12
    d1 = oracle.rope(q, 37, 1e7) @ oracle.rope(k, 30, 1e7)
    d2 = oracle.rope(q, 1007, 1e7) @ oracle.rope(k, 1000, 1e7)
    assert abs(d1 - d2) < 1e-10


def test_rope_pair_rotation_brute_force():
    D, pos, theta = 8, 3, 10000.0
    x = rng.standard_normal(D)
    y = oracle.rope(x, pos, theta)
    for i in range(D // 2):
        ang = pos * theta ** (-2 * i / D)
        assert abs(y[i] - (x[i] * math.cos(ang) - x[i + D // 2] * math.sin(ang))) < 1e-14
        assert abs(y[i + D // 2] - (x[i] * math.sin(ang) + x[i + D // 2] * math.cos(ang))) < 1e-14


def test_attention_single_position_returns_v():
    q = rng.standard_normal((4, 8))
    K = rng.standard_normal((2, 1, 8))
    V = rng.standard_normal((2, 1, 8))
    o = oracle.attention_decode(q, K, V)
    for h in range(4):
        np.testing.assert_allclose(o[h], V[h // 2, 0], rtol=1e-15)


def test_attention_brute_force_gqa():
    Hq, Hkv, P, D = 4, 2, 5, 3
    q = rng.standard_normal((Hq, D))
    K = rng.standard_normal((Hkv, P, D))
    V = rng.standard_normal((Hkv, P, D))
    o = oracle.attention_decode(q, K, V)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        s = [sum(q[h][d] * K[g][j][d] for d in range(D)) / math.sqrt(D) for j in range(P)]
        e = [math.exp(v) for v in s]
        z = sum(e)
        ref = [sum(e[j] / z * V[g][j][d] for j in range(P)) for d in range(D)]
        np.testing.assert_allclose(o[h], ref, rtol=1e-12)


def test_attention_split_combine_equals_unsplit():
    """Flash-decoding combine of per-split (m, l, acc) equals the one-pass softmax."""
    P, D = 50, 8
    q = rng.standard_normal(D)
    K = rng.standard_normal((P, D))
    V = rng.standard_normal((P, D))
    full = oracle.attention_decode(q[None], K[None], V[None])[0]
    parts = []
    for s in range(0, P, 16):
        sc = K[s:s + 16] @ q / math.sqrt(D)
        m = sc.max()
        parts.append((m, np.exp(sc - m).sum(), np.exp(sc - m) @ V[s:s + 16]))
    M = max(p[0] for p in parts)
    L = sum(p[1] * math.exp(p[0] - M) for p in parts)
    acc = sum(p[2] * math.exp(p[0] - M) for p in parts)
    np.testing.assert_allclose(acc / L, full, rtol=1e-12)


def test_log_softmax_brute_force():
    z = rng.standard_normal(7) * 5
    lse = math.log(sum(math.exp(v) for v in z))
    np.testing.assert_allclose(oracle.log_softmax(z), [v - lse for v in z], rtol=1e-13)
