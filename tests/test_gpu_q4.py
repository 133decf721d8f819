"""Q4_K-style weights in the decode megakernel, through the C ABI, against the oracle
(which dequantises the same 144-byte super-blocks exactly in float64).

Every 2-D projection, the tied embedding / LM head included, is 4-bit; conv taps and
RMSNorm gains stay bf16. The out- and down-projections run split over output rows on the
staged mixer output / activation.
"""
import numpy as np
import pytest

import oracle
import synth
from parity_util import LOGIT_MAX_ABS, MEAN_KL, STATE_REL_FROB, conv_history_as_window, kl, near_tie, rel_frob

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _setup(cfg, max_ctx, max_draft=0):
    import hybrid_deltanet_attention_b200 as hda
    raw = synth.make_weights(cfg)
    m = hda.Model(cfg, hda.weights_to_device(raw), max_ctx=max_ctx, max_draft=max_draft)
    return m, oracle.prepare_weights(cfg, raw)


def _teacher_forced(cfg, m, W, n_prompt, n_gen, max_ctx):
    dev = torch.device("cuda")
    m.reset()
    st = oracle.new_state(cfg, max_ctx)
    prompt = synth.make_prompt(cfg, n_prompt, tag="q4")
    z = oracle.prefill(cfg, W, st, prompt)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device=dev)
    nxt = torch.empty(1, dtype=torch.int32, device=dev)
    m.prefill(torch.from_numpy(prompt).to(dev), logits=logits, next_token=nxt)
    zo, zg, tg = [z], [logits.double().cpu().numpy()], [int(nxt.item())]
    tok = int(np.argmax(z))
    tin = torch.tensor([tok], dtype=torch.int32, device=dev)
    for _ in range(n_gen):
        m.decode(tin, nxt, logits)
        z = oracle.decode_step(cfg, W, st, tok)
        zo.append(z)
        zg.append(logits.double().cpu().numpy())
        tg.append(int(nxt.item()))
        tok = int(np.argmax(z))
        tin.fill_(tok)
    assert m.sync() == 0
    zo, zg = np.stack(zo), np.stack(zg)
    assert np.abs(zo - zg).max() <= LOGIT_MAX_ABS, np.abs(zo - zg).max()
    agree = np.argmax(zo, axis=1) == np.array(tg)
    ties = np.array([near_tie(z) for z in zo])
    assert agree[~ties].all()
    assert kl(zo, zg).mean() <= MEAN_KL
    S = m.S.cpu().numpy()
    assert max(rel_frob(S[li], st.S[li]) for li in range(cfg.n_dn)) <= STATE_REL_FROB
    ring = m.conv_history.cpu().numpy()
    for li in range(cfg.n_dn):
        assert rel_frob(conv_history_as_window(ring[li], st.pos, cfg.conv_width), st.conv[li]) <= STATE_REL_FROB
    assert int(m.pos_tensor.item()) == st.pos


def test_tiny_q4_decode_parity():
    cfg = synth.TINY_Q4
    m, W = _setup(cfg, 64)
    _teacher_forced(cfg, m, W, 20, 12, 64)


def test_mid_q4_decode_parity():
    cfg = synth.MID_Q4
    m, W = _setup(cfg, 64)
    _teacher_forced(cfg, m, W, 10, 6, 64)


def test_tiny_q4_verify_matches_oracle():
    cfg = synth.TINY_Q4
    m, W = _setup(cfg, 128, max_draft=5)
    dev = torch.device("cuda")
    K = 5
    prompt = synth.make_prompt(cfg, 12, tag="q4v")
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
        last = int(committed[-1])


def test_mid_q4_batched_prefill_two_passes():
    """A 70-token prompt on the mid-size 4-bit model: two batched passes (64 + 6 tokens,
    4-bit linear layers on 8-token tiles), then the last token's logits from its residual row."""
    cfg = synth.MID_Q4
    m, W = _setup(cfg, 128)
    _teacher_forced(cfg, m, W, 70, 2, 128)


def test_mid_q4_verify_one_pass():
    """Speculative verify with 4-bit weights: K + 1 tokens in one pass over the weights,
    acceptance and the DeltaNet state committed to the accepted prefix."""
    cfg = synth.MID_Q4
    m, W = _setup(cfg, 128, max_draft=5)
    dev = torch.device("cuda")
    K = 5
    prompt = synth.make_prompt(cfg, 24, tag="q4mv")
    m.reset()
    st = oracle.new_state(cfg, 128)
    oracle.prefill(cfg, W, st, prompt[:-1])
    m.prefill(torch.from_numpy(prompt[:-1]).to(dev))
    last = int(prompt[-1])
    for ps in range(2):
        greedy, _ = oracle.greedy_generate(cfg, W, st.copy(), last, K)
        use, ids = synth.draft_choices(4, ps, K, cfg.vocab)
        if ps == 0:
            use[:] = True
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
        assert int(m.pos_tensor.item()) == st.pos
        last = int(committed[-1])


@pytest.fixture(scope="module")
def q27():
    """Four layers of the 27B shape (hidden 5120, 48 DeltaNet heads, 24/4 attention heads,
    FFN 17408, seed-4 4-bit weights) with a 32K vocabulary."""
    cfg = synth.QWEN_27B_4L_32K
    m, W = _setup(cfg, 96, max_draft=5)
    return cfg, m, W


def test_27b_shape_q4_decode_parity(q27):
    """The hidden-5120 decode instance the 27B model runs (prompt through decode launches,
    then teacher-forced steps), against the oracle."""
    cfg, m, W = q27
    _teacher_forced(cfg, m, W, 8, 6, 96)


def test_27b_shape_q4_batched_prefill_and_verify(q27):
    """A 40-token prompt through the batched 4-bit prefill, then two verify passes of five
    drafts (all right, then the seeded mix), against the oracle."""
    cfg, m, W = q27
    dev = torch.device("cuda")
    K = 5
    prompt = synth.make_prompt(cfg, 41, tag="q27v")
    m.reset()
    st = oracle.new_state(cfg, 96)
    oracle.prefill(cfg, W, st, prompt[:-1])
    m.prefill(torch.from_numpy(prompt[:-1]).to(dev))
    last = int(prompt[-1])
    for ps in range(2):
        greedy, _ = oracle.greedy_generate(cfg, W, st.copy(), last, K)
        use, ids = synth.draft_choices(4, ps, K, cfg.vocab)
        if ps == 0:
            use[:] = True
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
        assert int(m.pos_tensor.item()) == st.pos
        last = int(committed[-1])
