"""Long-context decode: the 0.8B-shaped model with a seeded 32768-position KV cache in
every attention layer and seeded DeltaNet states, through the C ABI, against the oracle.

The state recipe is the long-context workload of the 0.8B hybrid: keys and values
i.i.d. N(0, 1) stored as bf16 with RoPE already applied, S i.i.d. N(0, 0.1), zero conv
tails, the next position 32768, and a uniform first token from seed 3. This exercises
the split-K attention path with the cache split over every CTA of the grid.
"""
import numpy as np
import pytest

import oracle
import synth
from parity_util import LOGIT_MAX_ABS, MEAN_KL, STATE_REL_FROB, kl, near_tie, rel_frob

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

N_POS = 32768
N_STEPS = 3


def _seed_both(cfg, m, max_ctx):
    ks, vs, ss = synth.long_context_state(cfg, N_POS)
    st = oracle.new_state(cfg, max_ctx)
    kc, vc, S = m.k_cache, m.v_cache, m.S
    for ai in range(cfg.n_at):
        kc[ai, :, :N_POS] = torch.from_numpy(ks[ai].view(np.int16)).to(kc.device).view(torch.bfloat16)
        vc[ai, :, :N_POS] = torch.from_numpy(vs[ai].view(np.int16)).to(vc.device).view(torch.bfloat16)
        st.K[ai][:, :N_POS] = oracle.decode_bf16_bits(ks[ai])
        st.V[ai][:, :N_POS] = oracle.decode_bf16_bits(vs[ai])
    for li in range(cfg.n_dn):
        S[li] = torch.from_numpy(ss[li]).to(S.device)
        st.S[li] = ss[li].astype(np.float64)
    m.set_position(N_POS)
    st.pos = N_POS
    return st


def test_08b_long_context_32k():
    import hybrid_deltanet_attention_b200 as hda
    cfg = synth.QWEN_08B
    dev = torch.device("cuda")
    max_ctx = N_POS + 8
    raw = synth.make_weights(cfg)
    m = hda.Model(cfg, hda.weights_to_device(raw), max_ctx=max_ctx)
    W = oracle.prepare_weights(cfg, raw)
    del raw
    m.reset()
    st = _seed_both(cfg, m, max_ctx)
    assert m.sync() == 0

    tok = int(synth.stream(3, "long.first_token").integers(0, cfg.vocab))
    tin = torch.tensor([tok], dtype=torch.int32, device=dev)
    tout = torch.empty(1, dtype=torch.int32, device=dev)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device=dev)
    zo, zg = [], []
    for _ in range(N_STEPS):
        m.decode(tin, tout, logits)
        assert m.sync() == 0
        z = oracle.decode_step(cfg, W, st, tok)
        zo.append(z)
        zg.append(logits.double().cpu().numpy())
        g = int(tout.item())
        assert g == int(np.argmax(zg[-1]))           # the kernel's token is its own logits' argmax
        if not near_tie(z):
            assert g == int(np.argmax(z))
        tok = int(np.argmax(z))                      # teacher forcing on the oracle's token
        tin.fill_(tok)
    zo, zg = np.stack(zo), np.stack(zg)
    assert np.abs(zo - zg).max() <= LOGIT_MAX_ABS, np.abs(zo - zg).max()
    assert kl(zo, zg).mean() <= MEAN_KL
    S = m.S.cpu().numpy()
    worst = max(rel_frob(S[li], st.S[li]) for li in range(cfg.n_dn))
    assert worst <= STATE_REL_FROB, worst
    # the appended keys and values of the new positions
    K = m.k_cache.float().cpu().numpy()
    V = m.v_cache.float().cpu().numpy()
    for ai in range(cfg.n_at):
        np.testing.assert_allclose(K[ai][:, N_POS:N_POS + N_STEPS], st.K[ai][:, N_POS:N_POS + N_STEPS],
                                   atol=2e-2, rtol=2e-2)
        np.testing.assert_allclose(V[ai][:, N_POS:N_POS + N_STEPS], st.V[ai][:, N_POS:N_POS + N_STEPS],
                                   atol=2e-2, rtol=2e-2)
        # the seeded part of the cache is untouched
        assert np.array_equal(K[ai][:, :N_POS], st.K[ai][:, :N_POS])
    assert int(m.pos_tensor.item()) == N_POS + N_STEPS
