"""Writes oracle_regression.json: a fingerprint of the oracle's outputs on seeded tiny-model
inputs, so that any later change to the oracle's arithmetic shows up in
tests/test_oracle_regression.py and has to be justified. Calls only `oracle` and `synth`.

    python tests/golden/make_oracle_regression.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_regression.json")


def fingerprint(z: np.ndarray) -> dict:
    top = np.argsort(-z, kind="stable")[:8]
    return {"top_index": [int(i) for i in top], "top_value": [float(z[i]) for i in top],
            "sum": float(z.sum()), "l2": float(np.sqrt((z * z).sum()))}


def compute() -> dict:
    cfg = synth.TINY
    W = oracle.prepare_weights(cfg, synth.make_weights(cfg))
    out = {}
    for name, kv_q8 in (("bf16_cache", False), ("q8_cache", True)):
        st = oracle.new_state(cfg, 64, kv_q8=kv_q8)
        z = oracle.prefill(cfg, W, st, synth.make_prompt(cfg, 16, seed=7))
        steps = [fingerprint(z)]
        tok = int(np.argmax(z))
        for _ in range(3):
            z = oracle.decode_step(cfg, W, st, tok)
            steps.append(fingerprint(z))
            tok = int(np.argmax(z))
        out[name] = {"steps": steps, "S_l2": [float(np.sqrt((s * s).sum())) for s in st.S], "pos": st.pos}
    u = np.random.default_rng(5).random((3, 2))
    logits = np.random.default_rng(6).standard_normal((3, 50))
    n, committed, margin = oracle.accept_sampled(logits, [int(np.argmax(logits[0])), 3], 0.7, u)
    out["accept_sampled"] = {"n": int(n), "committed": [int(c) for c in committed], "margin": float(margin)}
    return out


if __name__ == "__main__":
    with open(OUT, "w") as fh:
        json.dump(compute(), fh, indent=1)
    print("wrote", OUT)
