"""Whole-model pins for the oracle: an independent plain-Python float64 model,
the plain definition of speculative verify, and the Q4_K-style decoder."""
import struct

import numpy as np
import pytest

import oracle
import synth
from pyref_model import PyModel

MINI = synth.MINI


@pytest.fixture(scope="module")
def mini():
    raw = synth.make_weights(MINI)
    return raw, oracle.prepare_weights(MINI, raw)


@pytest.mark.parametrize("act", [False, True])
def test_oracle_matches_independent_python_model(mini, act):
    raw, W = mini
    py = PyModel(MINI, raw)
    st = oracle.new_state(MINI, 32)
    toks = [3, 17, 60, 0, 41, 41, 9]
    for t in toks:
        z_or = oracle.decode_step(MINI, W, st, t, act_bf16=act)
        z_py = np.array(py.step(t, act))
        np.testing.assert_allclose(z_or, z_py, rtol=1e-9, atol=1e-12)
    # states too
    for li in range(MINI.n_dn):
        np.testing.assert_allclose(st.S[li], np.array(py.S[li]), rtol=1e-9, atol=1e-12)


def test_mini_gated_and_tiny_ungated_shapes(mini):
    raw = synth.make_weights(synth.TINY)
    assert raw["layers.3.attn.w_in"].shape == ((4 + 2) * 64, 256)   # no gate rows in the tiny model
    assert raw["layers.3.attn.w_in"].shape[0] == synth.TINY.at_in_rows
    assert mini[0]["layers.3.attn.w_in"].shape[0] == (2 * 2 + 2) * 8


def test_prefill_equals_repeated_decode(mini):
    _, W = mini
    toks = synth.make_prompt(MINI, 9)
    a = oracle.new_state(MINI, 32)
    za = oracle.prefill(MINI, W, a, toks)
    b = oracle.new_state(MINI, 32)
    for t in toks:
        zb = oracle.decode_step(MINI, W, b, int(t))
    np.testing.assert_array_equal(za, zb)
    assert a.pos == b.pos == 9


def _states_equal(a, b):
    assert a.pos == b.pos
    for x, y in zip(a.S + a.conv + a.K + a.V, b.S + b.conv + b.K + b.V):
        np.testing.assert_array_equal(x, y)


def test_verify_exactness(mini):
    _, W = mini
    prompt = synth.make_prompt(MINI, 6)
    base = oracle.new_state(MINI, 64)
    z = oracle.prefill(MINI, W, base, prompt[:-1])
    last = int(prompt[-1])
    # plain greedy continuation from this state
    g_state = base.copy()
    greedy, _ = oracle.greedy_generate(MINI, W, g_state, last, 6)
    K = 5
    # all drafts right -> K + 1 tokens, identical to greedy
    st = base.copy()
    n, committed, logits = oracle.verify_drafts(MINI, W, st, last, greedy[:K])
    assert n == K and list(committed) == list(greedy[:K + 1])
    ref = base.copy()
    for t in [last] + list(greedy[:K]):
        oracle.decode_step(MINI, W, ref, int(t))
    _states_equal(st, ref)
    # all drafts wrong -> one token and the state equals one decode step
    wrong = [(int(g) + 1) % MINI.vocab for g in greedy[:K]]
    st = base.copy()
    n, committed, _ = oracle.verify_drafts(MINI, W, st, last, wrong)
    assert n == 0 and list(committed) == [greedy[0]]
    ref = base.copy()
    oracle.decode_step(MINI, W, ref, last)
    _states_equal(st, ref)
    # a mix: the second draft wrong
    mix = [int(greedy[0]), (int(greedy[1]) + 3) % MINI.vocab, 1, 2, 3]
    st = base.copy()
    n, committed, _ = oracle.verify_drafts(MINI, W, st, last, mix)
    assert n == 1 and list(committed) == [greedy[0], greedy[1]]


def test_drafts_compose():
    use, ids = synth.draft_choices(5, 0, 64, 100)
    greedy = np.arange(64, dtype=np.int32) % 100
    d = synth.compose_drafts(greedy, use, ids, 100)
    assert np.all(d[use] == greedy[use])
    assert np.all(d[~use] != greedy[~use])
    assert 0.6 < use.mean() < 0.95


# ------------------------------------------------------------------ Q4_K-style blocks
def _hand_block(d_bits, dmin_bits, sc, m, q):
    """Pack one block from its fields by the byte-layout definition (independent of synth)."""
    blk = bytearray(144)
    blk[0:2] = struct.pack("<H", d_bits)
    blk[2:4] = struct.pack("<H", dmin_bits)
    stream = 0
    for f, v in enumerate(list(sc) + list(m)):
        stream |= (v & 0x3F) << (6 * f)
    blk[4:16] = stream.to_bytes(12, "little")
    for j in range(8):
        for t in range(16):
            blk[16 + 16 * j + t] = q[32 * j + t] | (q[32 * j + t + 16] << 4)
    return np.frombuffer(bytes(blk), dtype=np.uint8)


def test_q4k_hand_built_block():
    # d = 0.5 (fp16 0x3800), dmin = 0.25 (fp16 0x3400); sc_j = j + 1, m_j = 2j, q_i = i mod 16
    sc = [j + 1 for j in range(8)]
    m = [2 * j for j in range(8)]
    q = [i % 16 for i in range(256)]
    blk = _hand_block(0x3800, 0x3400, sc, m, q)
    want = [0.5 * sc[i // 32] * q[i] - 0.25 * m[i // 32] for i in range(256)]
    np.testing.assert_array_equal(oracle.dequant_q4k_block(blk), want)
    np.testing.assert_array_equal(oracle.dequant_q4k_matrix(blk[None, :], 256)[0], want)
    # extreme fields: all 63, codes 15
    blk = _hand_block(0x3C00, 0x3C00, [63] * 8, [63] * 8, [15] * 256)   # d = dmin = 1
    np.testing.assert_array_equal(oracle.dequant_q4k_block(blk), [63 * 15 - 63] * 256)


def test_q4k_quantize_roundtrip_bound():
    r = np.random.default_rng(3)
    w = (r.standard_normal((6, 512)) * 0.02).astype(np.float32)
    data = synth.quantize_q4k(w)
    assert data.shape == (6, 2 * 144)
    deq = oracle.dequant_q4k_matrix(data, 512)
    for row in range(6):
        for blk in range(2):
            d, dmin, sc, m, q = oracle.unpack_q4k_fields(data[row, blk * 144:(blk + 1) * 144])
            for j in range(8):
                step = d * sc[j]
                sl = slice(blk * 256 + 32 * j, blk * 256 + 32 * j + 32)
                err = np.abs(deq[row, sl] - w[row, sl])
                inner = (q[32 * j:32 * j + 32] > 0) & (q[32 * j:32 * j + 32] < 15)
                assert np.all(err[inner] <= 0.5 * step * (1 + 1e-6) + 1e-9)
                # clipped codes: bounded by the sub-block's range (scale rounding is at most 1/126 relative)
                assert np.all(err <= 0.6 * step + 0.02 * (w[row, sl].max() - w[row, sl].min()) + 1e-6)
    # overall the 4-bit model stays close to the fp32 draw
    assert np.abs(deq - w).mean() < 0.002
