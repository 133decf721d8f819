"""Batched prefill of the 0.8B-shaped model at the benchmark's prompt lengths (520 and
4096 tokens, from a fresh state) against the oracle's prefill of the same prompts.

These are the paths the timed prefill workloads take: the persistent tcgen05 linear
layers over hundreds of tiles (several tiles per CTA with both TMEM accumulators), the
SwiGLU epilogue, the chunked delta rule's tensor-core state pass over 9 and 64 chunks,
the attention GEMMs over up to 4096 keys with the causal softmax between them, and the
conv history and KV carry-over. The oracle runs the prompt layer by layer (its form
pinned equal to the token-by-token prefill) with the chunked delta rule (pinned equal to
the recurrence), so 4096 tokens take seconds instead of minutes.

Compared: the last position's logits (max-abs error, greedy token unless a near tie),
every DeltaNet layer's state (relative Frobenius), the conv history, every KV cache
entry written (bf16 within one step of the oracle's rounding, see parity_util), and the
device position.
"""
import numpy as np
import pytest

import oracle
import synth
from parity_util import (LOGIT_MAX_ABS, STATE_REL_FROB, assert_bf16_cache_close, conv_history_as_window, near_tie,
                         rel_frob)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

MAX_CTX = 4096 + 64


@pytest.fixture(scope="module")
def m08():
    import hybrid_deltanet_attention_b200 as hda
    cfg = synth.QWEN_08B
    raw = synth.make_weights(cfg)
    m = hda.Model(cfg, hda.weights_to_device(raw), max_ctx=MAX_CTX)
    W = oracle.prepare_weights(cfg, raw)
    del raw
    return cfg, m, W


@pytest.mark.parametrize("n", [520, 4096])
def test_08b_prefill_at_bench_lengths(m08, n):
    cfg, m, W = m08
    dev = torch.device("cuda")
    prompt = synth.make_prompt(cfg, n, tag=f"pp{n}")
    m.reset()
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device=dev)
    nxt = torch.empty(1, dtype=torch.int32, device=dev)
    m.prefill(torch.from_numpy(prompt).to(dev), logits=logits, next_token=nxt)
    assert m.sync() == 0
    st = oracle.new_state(cfg, MAX_CTX)
    zo = oracle.prefill_sequence(cfg, W, st, prompt, chunk=64)

    zg = logits.double().cpu().numpy()
    err = float(np.abs(zo - zg).max())
    assert err <= LOGIT_MAX_ABS, err
    if not near_tie(zo):
        assert int(nxt.item()) == int(np.argmax(zo))
    assert int(m.pos_tensor.item()) == n == st.pos
    S = m.S.cpu().numpy()
    worst = max(rel_frob(S[li], st.S[li]) for li in range(cfg.n_dn))
    assert worst <= STATE_REL_FROB, worst
    ring = m.conv_history.cpu().numpy()
    for li in range(cfg.n_dn):
        e = rel_frob(conv_history_as_window(ring[li], n, cfg.conv_width), st.conv[li])
        assert e <= STATE_REL_FROB, (li, e)
    K = m.k_cache.float().cpu().numpy()
    V = m.v_cache.float().cpu().numpy()
    for ai in range(cfg.n_at):
        assert_bf16_cache_close(K[ai][:, :n], st.K[ai][:, :n])
        assert_bf16_cache_close(V[ai][:, :n], st.V[ai][:, :n])
