"""The allocation-free decode step (scratch in a static device array of the library)
gives the same results as the ordinary decode step.

Callers that cannot allocate device memory where they step the model (real-time loops
that must not stall on cudaMalloc's implicit synchronisation, hosts with a fixed
device-memory budget) use mk_decode_step_noalloc. This test calls it through the C ABI
twice in a row and compares each call with mk_decode_step started from the same state:
logits, next token, and the whole state the step writes (DeltaNet states, the conv
history slot of the position, the KV cache row at the position, the position). It also
checks the refusal when the context is full. It is collected last so that a failure
here does not stop the rest of the suite, and it needs nothing from the other tests.
"""
import ctypes as C

import numpy as np
import pytest

import synth
from parity_util import LOGIT_MAX_ABS, STATE_REL_FROB, assert_bf16_cache_close, near_tie, rel_frob

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _noalloc(m, tok, out, logits):
    stream = torch.cuda.current_stream().cuda_stream
    return m.lib.mk_decode_step_noalloc(m.h, tok.data_ptr(), out.data_ptr(),
                                        None if logits is None else logits.data_ptr(), C.c_void_p(stream))


@pytest.mark.parametrize("name", ["tiny", "0.8b"])
def test_noalloc_step_matches_regular_step(name):
    import hybrid_deltanet_attention_b200 as hda
    cfg = synth.CONFIGS[name]
    dev = torch.device("cuda")
    m = hda.Model(cfg, hda.weights_to_device(synth.make_weights(cfg)), max_ctx=64)
    prompt = torch.from_numpy(synth.make_prompt(cfg, 9, tag="noalloc")).to(dev)
    tok = torch.empty(1, dtype=torch.int32, device=dev)
    m.prefill(prompt, next_token=tok)
    assert m.sync() == 0
    pos = 9
    for call in range(2):
        snap = m.state.clone()
        out_a = torch.empty(1, dtype=torch.int32, device=dev)
        lg_a = torch.empty(cfg.vocab, dtype=torch.float32, device=dev)
        m.decode(tok, out_a, lg_a)
        assert m.sync() == 0
        S_a = m.S.cpu().numpy()
        conv_a = m.conv_history.cpu().numpy()
        K_a = m.k_cache.float().cpu().numpy()
        V_a = m.v_cache.float().cpu().numpy()
        # back to the same starting state, then the allocation-free step
        m.state.copy_(snap)
        m.set_position(pos)
        out_b = torch.empty(1, dtype=torch.int32, device=dev)
        lg_b = torch.empty(cfg.vocab, dtype=torch.float32, device=dev)
        rc = _noalloc(m, tok, out_b, lg_b)
        assert rc == 0, m.lib.mk_last_error()
        assert m.sync() == 0
        za, zb = lg_a.cpu().numpy(), lg_b.cpu().numpy()
        assert np.abs(za - zb).max() <= LOGIT_MAX_ABS, (call, np.abs(za - zb).max())
        if not near_tie(za.astype(np.float64)):
            assert int(out_a.item()) == int(out_b.item())
        assert rel_frob(m.S.cpu().numpy(), S_a) <= STATE_REL_FROB
        conv_b = m.conv_history.cpu().numpy()
        for li in range(cfg.n_dn):
            assert rel_frob(conv_b[li], conv_a[li]) <= STATE_REL_FROB, li
        K_b = m.k_cache.float().cpu().numpy()
        V_b = m.v_cache.float().cpu().numpy()
        for ai in range(cfg.n_at):      # every row up to and including the one this step wrote
            assert_bf16_cache_close(K_b[ai][:, :pos + 1], K_a[ai][:, :pos + 1])
            assert_bf16_cache_close(V_b[ai][:, :pos + 1], V_a[ai][:, :pos + 1])
        assert int(m.pos_tensor.item()) == pos + 1
        pos += 1
        tok = out_b.clone()


def test_noalloc_step_refuses_a_full_context():
    """With every position of the context used, the call returns MK_ERR_CAPACITY before
    launching anything, and the state is left as it was."""
    import hybrid_deltanet_attention_b200 as hda
    cfg = synth.TINY
    dev = torch.device("cuda")
    m = hda.Model(cfg, hda.weights_to_device(synth.make_weights(cfg)), max_ctx=20)
    prompt = torch.from_numpy(synth.make_prompt(cfg, 20, tag="noalloc-full")).to(dev)
    m.prefill(prompt)
    assert m.sync() == 0
    before = m.state.clone()
    tok = torch.ones(1, dtype=torch.int32, device=dev)
    out = torch.empty(1, dtype=torch.int32, device=dev)
    assert _noalloc(m, tok, out, None) == hda._abi.MK_ERR_CAPACITY
    assert m.sync() == 0
    assert torch.equal(m.state, before)
