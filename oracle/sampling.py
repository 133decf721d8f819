"""Sampling-mode speculative verify by its plain definition, float64 numpy.

Test infrastructure only (see the package docstring).

Source: the open-jet Qwen3.8-27B megakernel follow-up post (speed section) says that
speculation changes no output: in greedy mode the tokens are those the model alone
would pick, and in sampling mode the tokens follow the model's own distribution.
The post gives no rule; the one written here is standard speculative
sampling (Leviathan, Kalman and Matias, "Fast Inference from Transformers via
Speculative Decoding", 2023; Chen et al., "Accelerating Large Language Model
Decoding with Speculative Sampling", 2023): a drafted token x drawn from q is kept
with probability min(1, p(x) / q(x)); at the first rejection the output token is
drawn from max(0, p - q), renormalised; if every draft is kept, one more token is
drawn from the target distribution after the last draft.

The verify call receives draft tokens, not draft distributions, so each draft is
a point mass (q = 1 at the drafted token d). The rule then reads: keep d with
probability p(d); on rejection, draw from p with d removed and the rest
renormalised.

Random numbers are inputs: uniforms[i, 0] decides the draft at position i
(kept iff uniforms[i, 0] < p_i(d_{i+1})), uniforms[i, 1] draws the output token
at position i by the inverse of the cumulative distribution (the smallest token
index whose cumulative probability exceeds it). p_i = softmax(logits_i / tau).
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from .model import OracleState, decode_step

__all__ = ["softmax_t", "inverse_cdf", "accept_sampled", "verify_drafts_sampled"]


def softmax_t(z: np.ndarray, tau: float) -> np.ndarray:
    """Target distribution softmax(z / tau) in float64."""
    if not tau > 0.0:
        raise ValueError("temperature must be positive")
    x = np.asarray(z, dtype=np.float64) / float(tau)
    x = x - x.max()
    w = np.exp(x)
    return w / w.sum()


def inverse_cdf(w: np.ndarray, r: float) -> Tuple[int, float]:
    """Smallest index j with sum(w[:j+1]) > r * sum(w), for weights w >= 0, sum > 0.

    Also returns the distance of r * sum(w) from the nearest cumulative boundary,
    divided by sum(w): below rounding level the chosen index is not unique.
    """
    w = np.asarray(w, dtype=np.float64)
    total = w.sum()
    if not total > 0.0:
        raise ValueError("no token has positive weight")
    cdf = np.cumsum(w) / total
    j = int(np.searchsorted(cdf, r, side="right"))
    if j >= len(w):                       # r at the very top: the last token with weight
        j = int(np.nonzero(w)[0][-1])
    lo = cdf[j - 1] if j > 0 else 0.0
    margin = min(abs(r - lo), abs(cdf[j] - r))
    return j, float(margin)


def accept_sampled(logits: np.ndarray, drafts, tau: float, uniforms: np.ndarray):
    """Sampled acceptance of one verify pass.

    logits [K+1, V]: row i is the model's output after input i of the pass
    ([last, d_1 .. d_K]), so row i scores the token at position i + 1.
    uniforms [K+1, 2] in [0, 1).
    Returns (n, committed tokens [n+1], margin): d_1..d_n followed by the drawn
    token; margin is the smallest distance of a uniform from the threshold it was
    compared against (probability units), i.e. how far the decision is from a tie.
    """
    drafts = [int(d) for d in drafts]
    K = len(drafts)
    logits = np.asarray(logits, dtype=np.float64)
    uniforms = np.asarray(uniforms, dtype=np.float64)
    assert logits.shape[0] == K + 1 and uniforms.shape == (K + 1, 2)
    margin = np.inf
    n = 0
    while n < K:
        p = softmax_t(logits[n], tau)
        d = drafts[n]
        pd = p[d] if 0 <= d < p.size else 0.0
        margin = min(margin, abs(uniforms[n, 0] - pd))
        if uniforms[n, 0] < pd:
            n += 1
            continue
        resid = p.copy()
        if 0 <= d < p.size:
            resid[d] = 0.0
        tok, m = inverse_cdf(resid, uniforms[n, 1])
        return n, np.array(drafts[:n] + [tok], dtype=np.int32), min(margin, m)
    p = softmax_t(logits[K], tau)
    tok, m = inverse_cdf(p, uniforms[K, 1])
    return K, np.array(drafts + [tok], dtype=np.int32), min(margin, m)


def verify_drafts_sampled(cfg, W, st: OracleState, last_tok: int, drafts, tau: float, uniforms,
                          act_bf16: bool = False, logits: Optional[np.ndarray] = None):
    """Sampled speculative verify of one pass on the oracle model.

    Scores [last_tok, d_1..d_K] on a copy of the state, takes the sampled
    acceptance above, then rebuilds the state from the original by feeding
    [last_tok, d_1..d_n] (the committed drafts; the drawn token is the next
    input, as in the greedy verify). With `logits` given, those scores are used
    instead of the oracle's own (to check a decision on another path's logits).
    Returns (n, committed tokens [n+1], logits [K+1, V], margin).
    """
    drafts = [int(d) for d in drafts]
    feed = [int(last_tok)] + drafts
    if logits is None:
        trial = st.copy()
        logits = np.stack([decode_step(cfg, W, trial, t, act_bf16) for t in feed])
    n, committed, margin = accept_sampled(logits, drafts, tau, uniforms)
    for t in feed[:n + 1]:
        decode_step(cfg, W, st, t, act_bf16)
    return n, committed, logits, margin
