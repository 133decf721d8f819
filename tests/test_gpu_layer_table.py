"""The decode megakernel's two-slot layer table, against the oracle.

When the per-CTA scratch of the decode kernel leaves no room for every layer's table entry
in shared memory, the kernel keeps two slots and loads layer l + 1's entry while it runs
layer l (the 64-layer 27B model takes this path). The two models here force it at a size
the float64 oracle steps in seconds; mk_query_sizes reports which form the kernel uses.
"""
import numpy as np
import pytest

import oracle
import synth
from parity_util import LOGIT_MAX_ABS, MEAN_KL, STATE_REL_FROB, assert_bf16_cache_close, conv_history_as_window, kl, near_tie, rel_frob

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_table_form_reported():
    import hybrid_deltanet_attention_b200 as hda
    for cfg, want in ((synth.TINY, synth.TINY.n_layers), (synth.QWEN_08B, synth.QWEN_08B.n_layers),
                      (synth.WIDE_GQA8, 2), (synth.WIDE_GQA8_Q4, 2), (synth.QWEN_27B, 2)):
        assert hda.query_sizes(cfg, max_ctx=64).layer_table_entries == want, cfg.name


@pytest.mark.parametrize("name,n_prompt", [("wide-gqa8", 20), ("wide-gqa8", 6), ("wide-gqa8-q4", 20)])
def test_two_slot_table_decode_parity(name, n_prompt):
    """A prompt (20 tokens: the batched prefill; 6: one decode launch per token), then
    teacher-forced decode steps, every one of them on the two-slot table: logits, greedy
    tokens, DeltaNet states, conv history, KV cache and position against the oracle."""
    import hybrid_deltanet_attention_b200 as hda
    cfg = synth.CONFIGS[name]
    max_ctx, n_gen = 64, 8
    raw = synth.make_weights(cfg)
    m = hda.Model(cfg, hda.weights_to_device(raw), max_ctx=max_ctx)
    assert m.sizes.layer_table_entries == 2
    W = oracle.prepare_weights(cfg, raw)
    dev = torch.device("cuda")
    st = oracle.new_state(cfg, max_ctx)
    prompt = synth.make_prompt(cfg, n_prompt, tag="ltab2")
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
    ties = np.array([near_tie(v) for v in zo])
    assert agree[~ties].all()
    assert kl(zo, zg).mean() <= MEAN_KL
    S = m.S.cpu().numpy()
    assert max(rel_frob(S[li], st.S[li]) for li in range(cfg.n_dn)) <= STATE_REL_FROB
    ring = m.conv_history.cpu().numpy()
    for li in range(cfg.n_dn):
        assert rel_frob(conv_history_as_window(ring[li], st.pos, cfg.conv_width), st.conv[li]) <= STATE_REL_FROB
    K = m.k_cache.float().cpu().numpy()
    V = m.v_cache.float().cpu().numpy()
    for ai in range(cfg.n_at):
        assert_bf16_cache_close(K[ai][:, :st.pos], st.K[ai][:, :st.pos])
        assert_bf16_cache_close(V[ai][:, :st.pos], st.V[ai][:, :st.pos])
    assert int(m.pos_tensor.item()) == st.pos
