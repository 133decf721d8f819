"""Prefill of a whole prompt, layer by layer, float64 numpy.

Test infrastructure only (see the package docstring).

A causal decoder maps a sequence to a sequence one layer at a time: every position
of layer l is computed before layer l + 1 starts. Each position still sees exactly
what it sees in the token-by-token step of ``model.decode_step`` (its own and the
earlier positions' keys, values and DeltaNet state), so the two orders give the same
numbers up to the order of float64 additions. This form is what makes the oracle fast
enough for prompts of thousands of tokens (one matrix product per projection and
layer instead of one matrix-vector product per token); its equality with the token-by-
token form is pinned on small models.

Sources for what is computed are those of ``model.py``: the Hacker News post on the
fused Qwen3.5-0.8B megakernel (design bullets: 18 DeltaNet and 6 attention layers,
attention = QKV, RoPE, causal softmax, output projection) and the Gated Delta Networks
recurrence S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t.
The DeltaNet mixer runs either the recurrence itself or its chunked (WY) form from
``chunked.py`` (Yang et al. 2024), which is pinned equal to the recurrence.
"""
from __future__ import annotations

import numpy as np

from .chunked import deltanet_chunked, deltanet_recurrent
from .kvq8 import q8_roundtrip
from .model import OracleState, l2norm, rmsnorm, round_bf16, sigmoid, silu, softplus

__all__ = ["prefill_sequence", "rope_positions", "causal_attention"]


def rope_positions(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotary embedding of x [T, H, D] where row t sits at positions[t].

    Half-split pairing (i, i + D/2), frequency theta^(-2i/D), angle = position * freq.
    """
    D = x.shape[-1]
    half = D // 2
    i = np.arange(half, dtype=np.float64)
    ang = np.asarray(positions, dtype=np.float64)[:, None, None] * theta ** (-2.0 * i / D)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def causal_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, pos0: int) -> np.ndarray:
    """Attention of T queries at positions pos0 .. pos0+T-1 over the cache.

    q: [T, Hq, D]; K, V: [Hkv, P, D] with P >= pos0 + T. Query head h reads kv head
    h // (Hq / Hkv); the query at position p sees keys 0..p. Scale 1 / sqrt(D).
    """
    T, Hq, D = q.shape
    Hkv = K.shape[0]
    grp = Hq // Hkv
    P = pos0 + T
    allowed = np.arange(P)[None, :] <= (pos0 + np.arange(T))[:, None]      # [T, P]
    out = np.empty((T, Hq, V.shape[-1]))
    for h in range(Hq):
        g = h // grp
        s = q[:, h, :] @ K[g, :P].T / np.sqrt(D)
        s = np.where(allowed, s, -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ V[g, :P]
    return out


def _deltanet_sequence(cfg, W, p, st: OracleState, li: int, X: np.ndarray, chunk):
    Hd, dk, dv, Wc = cfg.dn_heads, cfg.dn_dk, cfg.dn_dv, cfg.conv_width
    C = cfg.dn_conv_channels
    T = X.shape[0]
    Z = X @ W[p + "dn.w_in"].T                                 # [T, q; k; v; alpha; beta]
    raw, alpha, beta = Z[:, :C], Z[:, C:C + Hd], Z[:, C + Hd:C + 2 * Hd]
    full = np.concatenate([st.conv[li], raw], axis=0)          # [W-1 + T, C], oldest first
    taps = W[p + "dn.conv"]                                    # [C, W]; column W-1 multiplies x_t
    y = np.zeros((T, C))
    for j in range(Wc):
        y += full[j:j + T] * taps[:, j]
    y = silu(y)
    st.conv[li] = full[T:]                                     # the last W-1 inputs
    q = l2norm(y[:, :Hd * dk].reshape(T, Hd, dk))
    k = l2norm(y[:, Hd * dk:2 * Hd * dk].reshape(T, Hd, dk))
    v = y[:, 2 * Hd * dk:].reshape(T, Hd, dv)
    a = np.exp(-softplus(alpha))
    b = sigmoid(beta)
    O = np.empty((T, Hd, dv))
    for h in range(Hd):
        if chunk:
            O[:, h], st.S[li][h] = deltanet_chunked(st.S[li][h], q[:, h], k[:, h], v[:, h], a[:, h], b[:, h], chunk)
        else:
            O[:, h], st.S[li][h] = deltanet_recurrent(st.S[li][h], q[:, h], k[:, h], v[:, h], a[:, h], b[:, h])
    return O.reshape(T, Hd * dv)


def _attention_sequence(cfg, W, p, st: OracleState, li: int, X: np.ndarray):
    Hq, Hkv, D = cfg.at_q_heads, cfg.at_kv_heads, cfg.at_head_dim
    T = X.shape[0]
    Z = X @ W[p + "attn.w_in"].T                               # [T, q; gate; k; v]
    off = 0
    q = Z[:, off:off + Hq * D].reshape(T, Hq, D); off += Hq * D
    if cfg.at_out_gate:
        g = Z[:, off:off + Hq * D]; off += Hq * D
    k = Z[:, off:off + Hkv * D].reshape(T, Hkv, D); off += Hkv * D
    v = Z[:, off:off + Hkv * D].reshape(T, Hkv, D)
    pos0 = st.pos
    positions = pos0 + np.arange(T)
    q = rope_positions(q, positions, cfg.rope_theta)
    k = rope_positions(k, positions, cfg.rope_theta)
    store = q8_roundtrip if st.kv_q8 else round_bf16
    st.K[li][:, pos0:pos0 + T] = store(k).transpose(1, 0, 2)
    st.V[li][:, pos0:pos0 + T] = store(v).transpose(1, 0, 2)
    o = causal_attention(q, st.K[li], st.V[li], pos0).reshape(T, Hq * D)
    if cfg.at_out_gate:
        o = o * sigmoid(g)
    return o


def prefill_sequence(cfg, W, st: OracleState, tokens, act_bf16: bool = False, chunk=None) -> np.ndarray:
    """Feed a prompt as one sequence; returns the logits after the last token.

    Same state update and result as ``model.prefill`` (token by token). chunk=None
    runs the DeltaNet recurrence; an integer runs its chunked (WY) form with chunks
    of that many tokens.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    T = tokens.shape[0]
    if T == 0:
        raise ValueError("empty prompt")
    if st.K and st.pos + T > st.K[0].shape[1]:
        raise ValueError("context capacity exceeded")
    rnd = round_bf16 if act_bf16 else (lambda x: x)
    eps = cfg.rms_eps
    H = W["embed"][tokens].copy()                              # [T, hidden]
    di = ai = 0
    for l, kind in enumerate(cfg.pattern):
        p = f"layers.{l}."
        X = rnd(rmsnorm(H, W[p + "norm1"], eps))
        if kind == "D":
            O = _deltanet_sequence(cfg, W, p, st, di, X, chunk); di += 1
            H = H + rnd(O) @ W[p + "dn.w_out"].T
        else:
            O = _attention_sequence(cfg, W, p, st, ai, X); ai += 1
            H = H + rnd(O) @ W[p + "attn.w_out"].T
        X = rnd(rmsnorm(H, W[p + "norm2"], eps))
        act = silu(X @ W[p + "mlp.w_gate"].T) * (X @ W[p + "mlp.w_up"].T)
        H = H + rnd(act) @ W[p + "mlp.w_down"].T
    st.pos += T
    x = rnd(rmsnorm(H[-1], W["norm_f"], eps))
    return W["embed"] @ x
