"""Batched prefill (tensor-core projections, chunked WY delta rule, causal attention)
through mk_prefill, against the oracle's token-by-token prefill.

Prompts longer than 16 tokens take the batched path for every token; the last token's
logits come from its residual row (final norm, one LM-head row, argmax). Shorter prompts run
through the decode kernel token by token. The lengths below cover one partial chunk,
exact chunks of 64, ragged tails, several chunks, and a second prefill that continues
from a non-empty state (conv history and KV cache carried over).
"""
import numpy as np
import pytest

import oracle
import synth
from parity_util import assert_bf16_cache_close, LOGIT_MAX_ABS, STATE_REL_FROB, conv_history_as_window, near_tie, rel_frob

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _model(cfg, max_ctx):
    import hybrid_deltanet_attention_b200 as hda
    raw = synth.make_weights(cfg)
    m = hda.Model(cfg, hda.weights_to_device(raw), max_ctx=max_ctx)
    return m, oracle.prepare_weights(cfg, raw)


@pytest.fixture(scope="module")
def tiny():
    cfg = synth.TINY
    m, W = _model(cfg, 512)
    return cfg, m, W


def _check(cfg, m, st, zo, zg, tok_g):
    err = np.abs(zo - zg).max()
    assert err <= LOGIT_MAX_ABS, err
    if not near_tie(zo):
        assert tok_g == int(np.argmax(zo))
    S = m.S.cpu().numpy()
    worst = max([rel_frob(S[li], st.S[li]) for li in range(cfg.n_dn)] + [0.0])
    assert worst <= STATE_REL_FROB, worst
    ring = m.conv_history.cpu().numpy()
    for li in range(cfg.n_dn):
        assert rel_frob(conv_history_as_window(ring[li], st.pos, cfg.conv_width), st.conv[li]) <= STATE_REL_FROB
    K = m.k_cache.float().cpu().numpy()
    V = m.v_cache.float().cpu().numpy()
    for ai in range(cfg.n_at):
        assert_bf16_cache_close(K[ai][:, :st.pos], st.K[ai][:, :st.pos])
        assert_bf16_cache_close(V[ai][:, :st.pos], st.V[ai][:, :st.pos])
    assert int(m.pos_tensor.item()) == st.pos


def _prefill_both(cfg, m, st, W, prompt):
    dev = torch.device("cuda")
    zo = oracle.prefill(cfg, W, st, prompt)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device=dev)
    nxt = torch.empty(1, dtype=torch.int32, device=dev)
    m.prefill(torch.from_numpy(prompt).to(dev), logits=logits, next_token=nxt)
    assert m.sync() == 0
    return zo, logits.double().cpu().numpy(), int(nxt.item())


@pytest.mark.parametrize("n", [17, 64, 65, 66, 130, 200])
def test_tiny_batched_prefill(tiny, n):
    cfg, m, W = tiny
    m.reset()
    st = oracle.new_state(cfg, 512)
    prompt = synth.make_prompt(cfg, n, tag=f"pf{n}")
    zo, zg, tg = _prefill_both(cfg, m, st, W, prompt)
    _check(cfg, m, st, zo, zg, tg)


def test_tiny_prefill_continues_from_state(tiny):
    cfg, m, W = tiny
    m.reset()
    st = oracle.new_state(cfg, 512)
    _prefill_both(cfg, m, st, W, synth.make_prompt(cfg, 40, tag="cont-a"))
    zo, zg, tg = _prefill_both(cfg, m, st, W, synth.make_prompt(cfg, 90, tag="cont-b"))
    _check(cfg, m, st, zo, zg, tg)


def test_tiny_prefill_then_decode(tiny):
    cfg, m, W = tiny
    dev = torch.device("cuda")
    m.reset()
    st = oracle.new_state(cfg, 512)
    zo, zg, tg = _prefill_both(cfg, m, st, W, synth.make_prompt(cfg, 100, tag="pd"))
    tok = int(np.argmax(zo))
    tin = torch.tensor([tok], dtype=torch.int32, device=dev)
    tout = torch.empty(1, dtype=torch.int32, device=dev)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device=dev)
    for _ in range(4):
        m.decode(tin, tout, logits)
        z = oracle.decode_step(cfg, W, st, tok)
        assert np.abs(z - logits.double().cpu().numpy()).max() <= LOGIT_MAX_ABS
        tok = int(np.argmax(z))
        tin.fill_(tok)
    assert m.sync() == 0
    _check(cfg, m, st, z, logits.double().cpu().numpy(), int(tout.item()))


def test_08b_batched_prefill_130():
    cfg = synth.QWEN_08B
    m, W = _model(cfg, 256)
    m.reset()
    st = oracle.new_state(cfg, 256)
    zo, zg, tg = _prefill_both(cfg, m, st, W, synth.make_prompt(cfg, 130, tag="pf08"))
    _check(cfg, m, st, zo, zg, tg)


def test_08b_verify_one_pass():
    """Speculative verify on the 0.8B shape: K + 1 tokens in one pass over the weights,
    acceptance, and the DeltaNet state committed to the accepted prefix."""
    import hybrid_deltanet_attention_b200 as hda
    cfg = synth.QWEN_08B
    raw = synth.make_weights(cfg)
    m = hda.Model(cfg, hda.weights_to_device(raw), max_ctx=128, max_draft=5)
    W = oracle.prepare_weights(cfg, raw)
    del raw
    dev = torch.device("cuda")
    K = 5
    prompt = synth.make_prompt(cfg, 40, tag="vf08")
    m.reset()
    st = oracle.new_state(cfg, 128)
    oracle.prefill(cfg, W, st, prompt[:-1])
    m.prefill(torch.from_numpy(prompt[:-1]).to(dev))
    last = int(prompt[-1])
    for ps in range(3):
        greedy, _ = oracle.greedy_generate(cfg, W, st.copy(), last, K)
        use, ids = synth.draft_choices(4, ps, K, cfg.vocab)
        if ps == 0:
            use[:] = True
        if ps == 1:
            use[:] = False
        drafts = synth.compose_drafts(greedy, use, ids, cfg.vocab)
        n_or, committed, z_or = oracle.verify_drafts(cfg, W, st, last, drafts)
        toks = torch.from_numpy(np.concatenate([[last], drafts]).astype(np.int32)).to(dev)
        n_acc = torch.zeros(1, dtype=torch.int32, device=dev)
        out = torch.full((K + 1,), -1, dtype=torch.int32, device=dev)
        logits = torch.empty((K + 1, cfg.vocab), dtype=torch.float32, device=dev)
        m.verify(toks, n_acc, out, logits)
        assert m.sync() == 0
        assert int(n_acc.item()) == n_or
        assert list(out.cpu().numpy()[:n_or + 1]) == list(committed)
        assert np.abs(logits.cpu().numpy() - z_or).max() <= LOGIT_MAX_ABS
        S = m.S.cpu().numpy()
        assert max(rel_frob(S[li], st.S[li]) for li in range(cfg.n_dn)) <= STATE_REL_FROB
        ring = m.conv_history.cpu().numpy()
        for li in range(cfg.n_dn):
            assert rel_frob(conv_history_as_window(ring[li], st.pos, cfg.conv_width), st.conv[li]) <= STATE_REL_FROB
        assert int(m.pos_tensor.item()) == st.pos
        last = int(committed[-1])


def test_flash_attention_sharp_scores_and_continued_prompts():
    """The tiny model with its query and key projections scaled by 16 (exact in bf16), so the
    attention scores span hundreds of units: within a query row a later key tile often beats
    the running maximum by far more than the flash kernel's rescale threshold, and rows of the
    same warp take different branches. A 199-token batched pass (two query tiles), then
    continued prompts of 71 and 65 tokens whose queries sit past earlier positions (up to six
    key tiles per row), against the oracle."""
    import hybrid_deltanet_attention_b200 as hda
    cfg = synth.TINY
    raw = synth.make_weights(cfg)
    for li, kind in enumerate(cfg.pattern):
        if kind != "A":
            continue
        name = f"layers.{li}.attn.w_in"
        w = raw[name].copy()
        qk = cfg.at_q_heads * cfg.at_head_dim * (2 if cfg.at_out_gate else 1) + cfg.at_kv_heads * cfg.at_head_dim
        vals = (w[:qk].astype(np.uint32) << 16).view(np.float32) * np.float32(16.0)
        w[:qk] = synth.f32_to_bf16_bits(vals)
        raw[name] = w
    m = hda.Model(cfg, hda.weights_to_device(raw), max_ctx=512)
    W = oracle.prepare_weights(cfg, raw)
    st = oracle.new_state(cfg, 512)
    m.reset()
    prompt = synth.make_prompt(cfg, 200 + 72 + 66, tag="sharp")
    o = 0
    for n in (200, 72, 66):   # batched passes of 199, 71 and 65 tokens, each ending in a decode launch
        zo, zg, tg = _prefill_both(cfg, m, st, W, prompt[o:o + n])
        _check(cfg, m, st, zo, zg, tg)
        o += n
