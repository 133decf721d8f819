"""GPU parity of the 8-bit KV cache against the oracle's 8-bit cache, through the C ABI.

The oracle stores each entry as its 8-bit read-back value (blocks of 32, fp16 scale,
float32 codes rounded to nearest even); re-quantising a read-back block gives back its
codes and scale, so the oracle's codes are recovered from its cache. The GPU's entries
come from float32 projections, the oracle's from float64 ones: a code may differ by one
where the quotient sits within rounding of a half-integer.
"""
import numpy as np
import pytest

import oracle
import synth
from parity_util import GREEDY_AGREE, LOGIT_MAX_ABS, MEAN_KL, STATE_REL_FROB, kl, rel_frob

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

MAX_CTX = 160


@pytest.fixture(scope="module")
def tiny_q8():
    import hybrid_deltanet_attention_b200 as hda
    cfg = synth.TINY
    raw = synth.make_weights(cfg)
    m = hda.Model(cfg, hda.weights_to_device(raw), max_ctx=MAX_CTX, max_draft=4, kv_format=hda._abi.MK_KV_Q8)
    assert m.sizes.kv_row_bytes == 80          # 64 codes + 2 fp16 scales, padded to 16 bytes
    return cfg, m, oracle.prepare_weights(cfg, raw)


def _check_codes(cfg, m, st):
    n = st.pos
    worst_scale = 0.0
    diff_frac = []
    for which, cache in (("k", st.K), ("v", st.V)):
        codes, scales = m.kv_q8_rows(which)
        for ai in range(cfg.n_at):
            q_or, d_or = oracle.quantize_q8(cache[ai][:, :n])
            dq = np.abs(codes[ai][:, :n].astype(np.int32) - q_or.astype(np.int32))
            assert dq.max() <= 1
            diff_frac.append(float((dq > 0).mean()))
            rs = np.abs(scales[ai][:, :n].astype(np.float64) - d_or.astype(np.float64)) / \
                np.maximum(d_or.astype(np.float64), 1e-30)
            worst_scale = max(worst_scale, float(rs.max()))
    assert max(diff_frac) <= 0.01
    assert worst_scale <= 2.0 ** -9


@pytest.mark.parametrize("n_prompt", [20, 80])     # few-token attention / attention as two GEMMs
def test_q8_prefill_then_decode_matches_oracle(tiny_q8, n_prompt):
    cfg, m, W = tiny_q8
    dev = torch.device("cuda")
    m.reset()
    st = oracle.new_state(cfg, MAX_CTX, kv_q8=True)
    prompt = synth.make_prompt(cfg, n_prompt, seed=41)
    z_or = oracle.prefill(cfg, W, st, prompt)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device=dev)
    nxt = torch.empty(1, dtype=torch.int32, device=dev)
    m.prefill(torch.from_numpy(prompt).to(dev), logits=logits, next_token=nxt)
    assert m.sync() == 0
    worst = float(np.abs(logits.cpu().numpy() - z_or).max())
    agree, kls = [], []
    tin = torch.empty(1, dtype=torch.int32, device=dev)
    tok = int(np.argmax(z_or))
    for _ in range(12):
        z_or = oracle.decode_step(cfg, W, st, tok)
        tin.fill_(tok)
        m.decode(tin, nxt, logits)
        z = logits.cpu().numpy()
        worst = max(worst, float(np.abs(z - z_or).max()))
        agree.append(int(np.argmax(z)) == int(np.argmax(z_or)))
        kls.append(kl(z_or, z))
        tok = int(np.argmax(z_or))
    assert m.sync() == 0
    assert worst <= LOGIT_MAX_ABS, worst
    assert np.mean(agree) >= GREEDY_AGREE
    assert np.mean(kls) <= MEAN_KL
    S = m.S.cpu().numpy()
    assert max(rel_frob(S[li], st.S[li]) for li in range(cfg.n_dn)) <= STATE_REL_FROB
    assert int(m.pos_tensor.item()) == st.pos
    _check_codes(cfg, m, st)


def test_q8_verify_pass_matches_oracle(tiny_q8):
    cfg, m, W = tiny_q8
    dev = torch.device("cuda")
    m.reset()
    st = oracle.new_state(cfg, MAX_CTX, kv_q8=True)
    prompt = synth.make_prompt(cfg, 24, seed=42)
    last = int(np.argmax(oracle.prefill(cfg, W, st, prompt)))
    m.prefill(torch.from_numpy(prompt).to(dev))
    g, _ = oracle.greedy_generate(cfg, W, st.copy(), last, 4)
    drafts = [int(g[0]), int(g[1]), (int(g[2]) + 3) % cfg.vocab, int(g[3])]
    n_or, committed, _ = oracle.verify_drafts(cfg, W, st, last, drafts)
    toks = torch.tensor([last] + drafts, dtype=torch.int32, device=dev)
    n_acc = torch.empty(1, dtype=torch.int32, device=dev)
    out = torch.empty(5, dtype=torch.int32, device=dev)
    m.verify(toks, n_acc, out)
    assert m.sync() == 0
    assert int(n_acc.item()) == n_or == 2
    assert list(out.cpu().numpy()[:n_or + 1]) == list(committed)
    assert int(m.pos_tensor.item()) == st.pos
    _check_codes(cfg, m, st)
