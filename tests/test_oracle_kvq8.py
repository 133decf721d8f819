"""Pins for the oracle's 8-bit KV-cache entries (blocks of 32, one fp16 scale each).

What fixes them, independently of the oracle's code:
  * a hand-built block whose scale is exactly 1 has codes written out here (ties to even);
  * a block scaled by a power of two scales its scale and keeps its codes;
  * the stored scale equals torch's float16 conversion of amax / 127 computed in float32;
  * the read-back error is within half a step plus the fp16 rounding of the scale;
  * all-zero blocks read back as zeros (no division by zero); blocks are independent;
  * on the model: single-position attention returns the read-back v, and the 8-bit cache
    moves the tiny model's logits by no more than its read-back error can explain.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def _block(vals):
    x = np.zeros(32)
    x[:len(vals)] = vals
    return x


def test_hand_built_block_codes():
    x = _block([127.0, -127.0, 0.5, 1.5, 2.5, -0.5, -1.5, 3.49, 3.51, 126.5, -126.5, 0.0])
    q, d = oracle.quantize_q8(x)
    assert d.shape == (1,) and float(d[0]) == 1.0
    want = [127, -127, 0, 2, 2, 0, -2, 3, 4, 126, -126, 0]
    assert list(q[:12]) == want
    assert np.all(q[12:] == 0)
    np.testing.assert_array_equal(oracle.dequantize_q8(q, d)[:12], want)


def test_power_of_two_scaling_keeps_codes():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(64)
    q1, d1 = oracle.quantize_q8(x)
    for e in (-7, 3):
        q2, d2 = oracle.quantize_q8(x * 2.0 ** e)
        np.testing.assert_array_equal(q1, q2)
        np.testing.assert_array_equal(d2.astype(np.float64), d1.astype(np.float64) * 2.0 ** e)


def test_scale_is_fp16_of_amax_over_127():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 128)) * np.array([1e-3, 0.1, 1.0, 7.0, 300.0])[:, None]
    _, d = oracle.quantize_q8(x)
    blocks = torch.from_numpy(x.astype(np.float32)).reshape(5, 4, 32)
    ref = (blocks.abs().amax(dim=-1) / 127.0).half()
    np.testing.assert_array_equal(d, ref.numpy())


def test_roundtrip_error_bound():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((200, 256)) * rng.uniform(0.01, 10, size=(200, 1))
    q, d = oracle.quantize_q8(x)
    back = oracle.dequantize_q8(q, d)
    x32 = x.astype(np.float32).astype(np.float64)
    step = np.abs(x32).reshape(200, 8, 32).max(axis=-1) / 127.0
    # half a step, plus 127 codes times the fp16 rounding of the scale (relative 2^-11)
    bound = step * (0.5 + 127 * 2.0 ** -11) * (1 + 1e-6)
    err = np.abs(back - x32).reshape(200, 8, 32).max(axis=-1)
    assert np.all(err <= bound)
    assert np.abs(q.astype(np.int32)).max() == 127


def test_zero_and_independent_blocks():
    x = np.concatenate([np.zeros(32), np.full(32, -3.0), np.zeros(32)])
    q, d = oracle.quantize_q8(x)
    assert list(d.astype(np.float64)) == [0.0, float(np.float16(np.float32(3.0) / np.float32(127.0))), 0.0]
    assert np.all(q[:32] == 0) and np.all(q[64:] == 0) and np.all(q[32:64] == -127)
    back = oracle.q8_roundtrip(x)
    assert np.all(back[:32] == 0) and np.all(np.isfinite(back))


def test_rejects_ragged_head_dim():
    with pytest.raises(ValueError):
        oracle.quantize_q8(np.ones(48))


def test_single_position_attention_returns_readback_v():
    rng = np.random.default_rng(3)
    Hq, Hkv, D = 4, 2, 64
    q = rng.standard_normal((Hq, D))
    k = oracle.q8_roundtrip(rng.standard_normal((Hkv, 1, D)))
    v = oracle.q8_roundtrip(rng.standard_normal((Hkv, 1, D)))
    o = oracle.attention_decode(q, k, v)
    for h in range(Hq):
        np.testing.assert_allclose(o[h], v[h // (Hq // Hkv), 0], rtol=0, atol=1e-15)


def test_model_with_q8_cache_stays_close_to_bf16_cache():
    cfg = synth.TINY
    W = oracle.prepare_weights(cfg, synth.make_weights(cfg))
    prompt = synth.make_prompt(cfg, 24, seed=31)
    st_b = oracle.new_state(cfg, 64)
    st_q = oracle.new_state(cfg, 64, kv_q8=True)
    z_b = oracle.prefill(cfg, W, st_b, prompt)
    z_q = oracle.prefill(cfg, W, st_q, prompt)
    assert st_q.kv_q8 and st_q.copy().kv_q8
    # the cache entries are the read-back values of the same inputs' 8-bit blocks ...
    for ai in range(cfg.n_at):
        for t in range(st_q.pos):
            np.testing.assert_array_equal(st_q.K[ai][:, t], oracle.q8_roundtrip(st_q.K[ai][:, t]))
    # ... and the logits move by far less than their spread
    assert np.abs(z_q - z_b).max() < 0.05 * z_b.std()
    assert int(np.argmax(z_q)) == int(np.argmax(z_b))


# ------------------------------------------------------------------ planted mistakes (CPU only)
def _quantize_truncating(x):                         # slip: codes truncated toward zero
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    b = x32.reshape(*x32.shape[:-1], -1, 32)
    d = (np.abs(b).max(axis=-1) / np.float32(127)).astype(np.float32)
    q = np.trunc(b / np.where(d > 0, d, 1)[..., None]).astype(np.int8)
    return q.reshape(x32.shape), d.astype(np.float16)


def _quantize_scale_from_first(x):                   # slip: scale from the first entry, not the block max
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    b = x32.reshape(*x32.shape[:-1], -1, 32)
    d = (np.abs(b[..., 0]) / np.float32(127)).astype(np.float32)
    q = np.clip(np.rint(b / np.where(d > 0, d, 1)[..., None]), -127, 127).astype(np.int8)
    return q.reshape(x32.shape), d.astype(np.float16)


@pytest.mark.parametrize("fn", [_quantize_truncating, _quantize_scale_from_first])
def test_planted_q8_mistake_is_caught(fn):
    x = _block([0.5, 127.0, -127.0, 1.5, 2.5, -0.5, 3.49, 3.51])   # the block maximum is not first
    q_ref, d_ref = oracle.quantize_q8(x)
    assert list(q_ref[:8]) == [0, 127, -127, 2, 2, 0, 3, 4] and float(d_ref[0]) == 1.0
    q, d = fn(x)
    assert not (np.array_equal(q, q_ref) and np.array_equal(d, d_ref))
