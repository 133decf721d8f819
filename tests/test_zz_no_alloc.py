"""The allocation-free decode step (scratch in a static device array of the library)
gives the same results as the ordinary decode step.

Callers that cannot allocate device memory where they step the model (CUDA host
callbacks, real-time loops, fixed-budget hosts) use mk_decode_step_noalloc. This test
calls it through the C ABI twice in a row and compares each call with mk_decode_step
started from the same state. It is collected last so that a failure here does not stop
the rest of the suite, and it needs nothing from the other tests.
"""
import ctypes as C

import numpy as np
import pytest

import synth
from parity_util import LOGIT_MAX_ABS, STATE_REL_FROB, near_tie, rel_frob

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "0.8b"])
def test_noalloc_step_matches_regular_step(name):
    import hybrid_deltanet_attention_b200 as hda
    cfg = synth.CONFIGS[name]
    dev = torch.device("cuda")
    m = hda.Model(cfg, hda.weights_to_device(synth.make_weights(cfg)), max_ctx=64)
    lib = m.lib
    stream = torch.cuda.current_stream().cuda_stream
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
        S_a = m.S.clone()
        # back to the same starting state, then the allocation-free step
        m.state.copy_(snap)
        m.set_position(pos)
        out_b = torch.empty(1, dtype=torch.int32, device=dev)
        lg_b = torch.empty(cfg.vocab, dtype=torch.float32, device=dev)
        rc = lib.mk_decode_step_noalloc(m.h, tok.data_ptr(), out_b.data_ptr(), lg_b.data_ptr(), C.c_void_p(stream))
        assert rc == 0, lib.mk_last_error()
        assert m.sync() == 0
        za, zb = lg_a.cpu().numpy(), lg_b.cpu().numpy()
        assert np.abs(za - zb).max() <= LOGIT_MAX_ABS, (call, np.abs(za - zb).max())
        if not near_tie(za.astype(np.float64)):
            assert int(out_a.item()) == int(out_b.item())
        assert rel_frob(m.S.cpu().numpy(), S_a.cpu().numpy()) <= STATE_REL_FROB
        assert int(m.pos_tensor.item()) == pos + 1
        pos += 1
        tok = out_b.clone()
