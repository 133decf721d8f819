"""GPU parity of the sampling-mode speculative verify against the CPU oracle, through the C ABI.

The uniforms are inputs (seeded here); every expected decision comes from ``oracle``:
on the kernel's own logits the decision must be identical unless a uniform lies within
rounding distance of its threshold (then the kernel's choice is checked for validity),
and on the oracle's logits it must agree whenever the margin exceeds what the logits
tolerance can move.
"""
import numpy as np
import pytest

import oracle
import synth
from parity_util import LOGIT_MAX_ABS, STATE_REL_FROB, rel_frob

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

KERNEL_MARGIN = 1e-9      # both sides decide in float64 from the same float32 logits
ORACLE_MARGIN = 1e-3      # logits within 3e-2 at temperature >= 0.15 on the tiny model (measured ~1e-5)


def _model(cfg, max_ctx, max_draft):
    import hybrid_deltanet_attention_b200 as hda
    raw = synth.make_weights(cfg)
    return hda.Model(cfg, hda.weights_to_device(raw), max_ctx=max_ctx, max_draft=max_draft), raw


def _run_pass(m, tokens, tau, u, V):
    dev = torch.device("cuda")
    K = len(tokens) - 1
    t = torch.tensor(tokens, dtype=torch.int32, device=dev)
    uu = torch.tensor(np.asarray(u, dtype=np.float32).reshape(-1), device=dev)
    n_acc = torch.full((1,), -1, dtype=torch.int32, device=dev)
    out = torch.full((K + 1,), -1, dtype=torch.int32, device=dev)
    logits = torch.empty((K + 1, V), dtype=torch.float32, device=dev)
    m.verify_sampled(t, tau, uu, n_acc, out, logits=logits)
    assert m.sync() == 0
    n = int(n_acc.item())
    return n, out.cpu().numpy()[:n + 1], logits.cpu().numpy().astype(np.float64), uu.cpu().numpy().astype(
        np.float64).reshape(K + 1, 2)


def _valid(n, committed, drafts, logits, tau):
    """What any correct run satisfies: kept drafts are a prefix, the drawn token has
    positive probability and is not the draft rejected at its position."""
    assert 0 <= n <= len(drafts)
    assert list(committed[:n]) == list(drafts[:n])
    p = oracle.softmax_t(logits[n], tau)
    tok = int(committed[n])
    assert 0 <= tok < p.size and p[tok] > 0.0
    if n < len(drafts):
        assert tok != drafts[n]


@pytest.fixture(scope="module")
def tiny():
    cfg = synth.TINY
    m, raw = _model(cfg, max_ctx=128, max_draft=5)
    return cfg, m, oracle.prepare_weights(cfg, raw)


@pytest.mark.parametrize("tau", [0.15, 0.6])
def test_sampled_verify_matches_oracle_tiny(tiny, tau):
    cfg, m, W = tiny
    dev = torch.device("cuda")
    rng = np.random.default_rng(int(tau * 1000))
    tau = float(np.float32(tau))       # the library takes the temperature as float32
    K = 4
    m.reset()
    st = oracle.new_state(cfg, 128)
    prompt = synth.make_prompt(cfg, 16, seed=21)
    z = oracle.prefill(cfg, W, st, prompt)
    m.prefill(torch.from_numpy(prompt).to(dev))
    last = int(np.argmax(z))          # both sides continue from the same token
    kept_total = strict = 0
    for it in range(10):
        g, _ = oracle.greedy_generate(cfg, W, st.copy(), last, K)
        drafts = [int(x) if rng.random() < 0.8 else int(rng.integers(cfg.vocab)) for x in g]
        u = rng.random((K + 1, 2))
        n, committed, lg, u = _run_pass(m, [last] + drafts, tau, u, cfg.vocab)   # u: the float32 values used
        _valid(n, committed, drafts, lg, tau)
        # the decision on the kernel's own logits
        n_k, c_k, margin_k = oracle.accept_sampled(lg, drafts, tau, u)
        if margin_k > KERNEL_MARGIN:
            strict += 1
            assert n == n_k and list(committed) == list(c_k), (it, n, n_k, committed, c_k)
        # the oracle's own scores and decision; its state follows the kernel's commit
        trial = st.copy()
        z_or = np.stack([oracle.decode_step(cfg, W, trial, t) for t in [last] + drafts])
        assert np.abs(lg - z_or).max() <= LOGIT_MAX_ABS
        n_o, c_o, margin_o = oracle.accept_sampled(z_or, drafts, tau, u)
        if margin_o > ORACLE_MARGIN:
            assert n == n_o and list(committed) == list(c_o)
        for t in [last] + drafts[:n]:
            oracle.decode_step(cfg, W, st, t)
        last = int(committed[n])
        kept_total += n
    assert strict >= 9
    assert kept_total < 10 * K          # rejections were exercised
    if tau < 0.2:
        assert kept_total > 0           # and so were kept drafts
    S = m.S.cpu().numpy()
    worst = max(rel_frob(S[li], st.S[li]) for li in range(cfg.n_dn))
    assert worst <= STATE_REL_FROB, worst
    assert int(m.pos_tensor.item()) == st.pos


def test_sampled_verify_low_temperature_equals_greedy_verify(tiny):
    cfg, m, W = tiny
    dev = torch.device("cuda")
    prompt = synth.make_prompt(cfg, 16, seed=22)
    rng = np.random.default_rng(5)
    K = 5
    results = []
    for mode in ("greedy", "sampled"):
        m.reset()
        m.prefill(torch.from_numpy(prompt).to(dev))
        st = oracle.new_state(cfg, 128)
        last = int(np.argmax(oracle.prefill(cfg, W, st, prompt)))
        g, _ = oracle.greedy_generate(cfg, W, st.copy(), last, K)
        drafts = [int(g[0]), int(g[1]), int(g[2]), (int(g[3]) + 7) % cfg.vocab, int(g[4])]
        t = torch.tensor([last] + drafts, dtype=torch.int32, device=dev)
        n_acc = torch.empty(1, dtype=torch.int32, device=dev)
        out = torch.empty(K + 1, dtype=torch.int32, device=dev)
        if mode == "greedy":
            m.verify(t, n_acc, out)
        else:
            uu = torch.tensor(rng.random(2 * (K + 1)).astype(np.float32), device=dev)
            m.verify_sampled(t, 1e-4, uu, n_acc, out)
        assert m.sync() == 0
        n = int(n_acc.item())
        results.append((n, list(out.cpu().numpy()[:n + 1]), m.S.cpu().numpy().copy()))
    assert results[0][0] == results[1][0] == 3
    assert results[0][1] == results[1][1]
    # same decisions, same commit; the states differ only by the order of float additions
    # in the split-K reductions of the two passes (measured 1.7e-6)
    assert rel_frob(results[1][2], results[0][2]) <= 1e-4


def test_sampled_verify_rejects_bad_arguments(tiny):
    cfg, m, W = tiny
    import hybrid_deltanet_attention_b200 as hda
    dev = torch.device("cuda")
    t = torch.zeros(3, dtype=torch.int32, device=dev)
    uu = torch.full((6,), 0.5, dtype=torch.float32, device=dev)
    n_acc = torch.empty(1, dtype=torch.int32, device=dev)
    out = torch.empty(3, dtype=torch.int32, device=dev)
    for tau in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(hda.MkError):
            m.verify_sampled(t, tau, uu, n_acc, out)
    t9 = torch.zeros(8, dtype=torch.int32, device=dev)         # K = 7 > max_draft
    with pytest.raises(hda.MkError):
        m.verify_sampled(t9, 1.0, torch.full((16,), 0.5, device=dev), n_acc, torch.empty(8, dtype=torch.int32,
                                                                                             device=dev))


def test_sampled_verify_full_vocab_08b():
    """0.8B shape (V = 151936, the launch configuration of the benchmarks): decisions on
    the kernel's logits, including the uniforms' extremes, which fix the draw exactly."""
    cfg = synth.QWEN_08B
    m, raw = _model(cfg, max_ctx=256, max_draft=5)
    dev = torch.device("cuda")
    prompt = synth.make_prompt(cfg, 32, seed=23)
    m.reset()
    nxt = torch.empty(1, dtype=torch.int32, device=dev)
    m.prefill(torch.from_numpy(prompt).to(dev), next_token=nxt)
    last = int(nxt.item())
    rng = np.random.default_rng(9)
    K = 5
    strict = 0
    for it in range(6):
        drafts = [int(x) for x in rng.integers(0, cfg.vocab, size=K)]
        u = rng.random((K + 1, 2))
        if it == 0:
            u[0, 0], u[0, 1] = 0.999, 0.0                  # reject d_1, then the first token with weight
        if it == 1:
            u[0, 0], u[0, 1] = 0.999, np.nextafter(np.float32(1), np.float32(0))   # ... the last one
        tau = 1.0 if it < 2 or it % 2 == 0 else float(np.float32(0.3))   # as the library receives it
        n, committed, lg, u = _run_pass(m, [last] + drafts, tau, u, cfg.vocab)
        _valid(n, committed, drafts, lg, tau)
        n_k, c_k, margin_k = oracle.accept_sampled(lg, drafts, tau, u)
        if it == 0:
            assert n == 0 and committed[0] == (1 if drafts[0] == 0 else 0)
        if it == 1:
            assert n == 0 and committed[0] == (cfg.vocab - 2 if drafts[0] == cfg.vocab - 1 else cfg.vocab - 1)
        if margin_k > KERNEL_MARGIN:
            strict += 1
            assert n == n_k and list(committed) == list(c_k), (it, n, n_k, committed, c_k)
        last = int(committed[n])
    assert strict >= 5
