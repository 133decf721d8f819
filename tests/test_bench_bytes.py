"""The roofline numerator: algorithmic bytes one decode step reads, pinned by a count made
by hand from the 0.8B-shaped architecture and by the loader's own tensor list."""
import numpy as np

import bench
import synth


def test_weights_equal_the_tensor_list():
    for cfg in (synth.TINY, synth.MINI, synth.QWEN_08B):
        specs = synth.tensor_specs(cfg)
        assert bench.bytes_per_token(cfg, 0)["weights"] == sum(int(np.prod(s)) for _, s, _ in specs) * 2


def test_08b_bytes_by_hand():
    cfg = synth.QWEN_08B
    H, V, F = 1024, 151936, 3584
    per_mlp = 2 * H + 3 * F * H                                    # two gains, gate, up, down
    per_dn = (3 * 16 * 128 + 2 * 16) * H + 3 * 16 * 128 * 4 + H * 16 * 128   # in-proj, conv taps, out-proj
    per_at = (8 * 256 + 8 * 256 + 2 * 256 + 2 * 256) * H + H * 8 * 256       # q, gate, k, v; out-proj
    weights = 2 * (V * H + H + 24 * per_mlp + 18 * per_dn + 6 * per_at)     # tied head + final gain
    b = bench.bytes_per_token(cfg, 191)
    assert b["weights"] == weights == 1_231_882_240
    assert b["state"] == 18 * 16 * 128 * 128 * 4                 # fp32 S of every DeltaNet layer
    assert b["kv"] == 6 * 2 * 256 * 2 * 2 * 192                  # bf16 K and V, positions 0..191
    assert b["kv"] == 12_288 * 192
    assert b["read"] == b["weights"] + b["state"] + b["conv"] + b["kv"]
    # about 1.255 GB a token at the tg128 positions: 192 us at the measured copy bandwidth
    assert 1.2548e9 < b["read"] < 1.2550e9


def test_08b_prefill_linear_macs_by_hand():
    H, F = 1024, 3584
    macs = 24 * 3 * F * H + 18 * (6176 * H + H * 2048) + 6 * (5120 * H + H * 2048)
    assert bench.linear_macs_per_token(synth.QWEN_08B) == macs == 459_866_112   # 0.92 GFLOP a token


def test_prefill_flops_by_hand():
    """The whole-prefill FLOP count the prefill line's roofline divides by, recounted by hand
    for a pp4096 prompt on the 0.8B shape: the linear layers of every token plus one LM-head
    row, causal attention over the keys each query sees, and the chunked delta rule (C = 64:
    K K^T, the lower triangles of Q K^T, of the solve for [U | W] and of P Delta, and Q S0^T,
    W S0^T and the state update)."""
    cfg = synth.QWEN_08B
    T, H, V = 4096, 1024, 151936
    f = bench.prefill_flops(cfg, T)
    assert f["linear"] == 2 * 459_866_112 * T + 2 * V * H
    keys = T * (T + 1) // 2                                      # query t sees keys 0..t
    assert f["attention"] == 6 * 8 * 2 * 2 * keys * 256          # 6 layers, 8 query heads, QK^T and PV
    C, dk, dv = 64, 128, 128
    per_token = C * dk + (C * dk) / 2 + (C * (dk + dv)) / 2 + 3 * dk * dv + (C * dv) / 2
    assert f["deltanet"] == 2 * per_token * 16 * 18 * T          # 16 heads, 18 DeltaNet layers
    assert abs(f["total"] - 4.354e12) < 0.001e12                 # ~4.35 TFLOP
    # a continued prompt attends to the cached positions too
    g = bench.prefill_flops(cfg, 64, pos0=100)
    assert g["attention"] == 6 * 8 * 2 * 2 * (64 * 100 + 64 * 65 // 2) * 256
