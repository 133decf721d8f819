"""Recurrent (token-by-token) forward step of the hybrid model, float64 numpy.

Test infrastructure only (see the package docstring).

Sources for what is computed:
  * Hacker News post on the fused 24-layer Qwen3.5-0.8B megakernel, design
    bullets: 18 of the 24 layers are DeltaNet mixers (linear attention whose
    state evolves by a learned recurrence), 6 are full attention; weights and
    activations are kept in bf16 and sums in fp32; attention = QKV, RoPE,
    causal softmax, output projection.
  * Gated DeltaNet (Yang, Kautz and Hatamizadeh, "Gated Delta Networks", 2024):
    S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t,
    with a_t = exp(-softplus(.)), b_t = sigmoid(.), L2-normalised q, k and a
    causal depthwise conv of width 4 with SiLU on the q/k/v channels.
  * Pre-norm residual blocks with RMSNorm and a SwiGLU MLP; the LM head is the
    tied embedding; greedy decoding takes the lowest index among equal maxima.
"""
from __future__ import annotations

import copy
import dataclasses
from typing import Dict, List, Optional

import numpy as np

from .kvq8 import q8_roundtrip

__all__ = [
    "round_bf16", "decode_bf16_bits", "rmsnorm", "silu", "sigmoid", "softplus", "l2norm",
    "conv_silu", "delta_rule_step", "rope", "attention_decode", "swiglu",
    "OracleState", "new_state", "prepare_weights", "decode_step", "prefill",
    "greedy_generate", "verify_drafts", "log_softmax",
]


# ------------------------------------------------------------------ scalars and vectors
def decode_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """bf16 bit pattern (uint16) -> float64 value (exact)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value, ties to even, returned as float64.

    Written from the IEEE definition: keep 8 significand bits. The fp64 value
    is first rounded to fp32 (its 24-bit significand holds every bf16 value),
    then to bf16 on the fp32 bit pattern; the two-step rounding differs from
    a direct one only for values within 2^-24 relative of a bf16 midpoint.
    """
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    out = (u.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return out.astype(np.float64)


def rmsnorm(h: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """x = h / sqrt(mean(h^2) + eps) * gamma (over the last axis)."""
    ms = np.mean(h * h, axis=-1, keepdims=True)
    return h / np.sqrt(ms + eps) * gamma


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    return x * sigmoid(x)


def softplus(x):
    """log(1 + e^x), evaluated as max(x, 0) + log1p(e^-|x|) so it never overflows."""
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def l2norm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(sum(x^2) + eps) over the last axis."""
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def log_softmax(z: np.ndarray) -> np.ndarray:
    m = np.max(z, axis=-1, keepdims=True)
    return z - m - np.log(np.sum(np.exp(z - m), axis=-1, keepdims=True))


# ------------------------------------------------------------------ mixers
def conv_silu(window: np.ndarray, x_t: np.ndarray, taps: np.ndarray) -> np.ndarray:
    """Causal depthwise conv of width W on one new input, then SiLU.

    window: [W-1, C] previous inputs, oldest first (zeros before the first token)
    x_t:    [C] current input;  taps: [C, W], column W-1 multiplies x_t.
    y[c] = SiLU( sum_j taps[c, j] * x_{t-(W-1)+j}[c] )
    """
    full = np.concatenate([window, x_t[None, :]], axis=0)      # [W, C]
    return silu(np.einsum("wc,cw->c", full, taps))


def delta_rule_step(S: np.ndarray, q: np.ndarray, k: np.ndarray, v: np.ndarray,
                    a: float, b: float):
    """One gated delta-rule step for one head.

    S_t = a S_{t-1} (I - b k k^T) + b v k^T   (S: [dv, dk]),  o = S_t q.
    Evaluated as written: decay, then the rank-1 correction toward v.
    """
    Sd = a * S
    S_new = Sd - b * np.outer(Sd @ k, k) + b * np.outer(v, k)
    return S_new, S_new @ q


def rope(x: np.ndarray, pos: int, theta: float) -> np.ndarray:
    """Rotary position embedding over the full head dim, half-split pairing.

    x: [..., D]; pairs (i, i + D/2), frequency theta^(-2i/D), angle = pos * freq.
    """
    D = x.shape[-1]
    half = D // 2
    i = np.arange(half, dtype=np.float64)
    ang = pos * theta ** (-2.0 * i / D)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def attention_decode(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Causal attention of the current token over positions 0..P-1.

    q: [Hq, D]; K, V: [Hkv, P, D]. Query head h reads kv head h // (Hq / Hkv).
    o_h = softmax(K_g q_h / sqrt(D)) V_g.
    """
    Hq, D = q.shape
    Hkv = K.shape[0]
    grp = Hq // Hkv
    out = np.empty((Hq, V.shape[-1]))
    for h in range(Hq):
        g = h // grp
        s = K[g] @ q[h] / np.sqrt(D)
        p = np.exp(s - s.max())
        p /= p.sum()
        out[h] = p @ V[g]
    return out


def swiglu(x: np.ndarray, w_gate, w_up) -> np.ndarray:
    return silu(w_gate @ x) * (w_up @ x)


# ------------------------------------------------------------------ weights and state
def prepare_weights(cfg, raw: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """Storage arrays (bf16 bits, or Q4_K-style bytes) -> float64 matrices."""
    from .q4k import dequant_q4k_matrix
    import synth
    W = {}
    for name, shape, _ in synth.tensor_specs(cfg):
        a = raw[name]
        if synth.is_quantized(cfg, name, shape):
            W[name] = dequant_q4k_matrix(a, shape[1])
        else:
            W[name] = decode_bf16_bits(a).reshape(shape)
    return W


@dataclasses.dataclass
class OracleState:
    S: List[np.ndarray]        # per DeltaNet layer [Hd, dv, dk]
    conv: List[np.ndarray]     # per DeltaNet layer [W-1, C] previous raw conv inputs, oldest first
    K: List[np.ndarray]        # per attention layer [Hkv, max_ctx, D] (bf16-valued, or q8 read-back values)
    V: List[np.ndarray]
    pos: int = 0
    kv_q8: bool = False        # 8-bit block entries (oracle/kvq8.py) instead of bf16

    def copy(self) -> "OracleState":
        return copy.deepcopy(self)


def new_state(cfg, max_ctx: int, kv_q8: bool = False) -> OracleState:
    S = [np.zeros((cfg.dn_heads, cfg.dn_dv, cfg.dn_dk)) for _ in range(cfg.n_dn)]
    conv = [np.zeros((cfg.conv_width - 1, cfg.dn_conv_channels)) for _ in range(cfg.n_dn)]
    shp = (cfg.at_kv_heads, max_ctx, cfg.at_head_dim)
    K = [np.zeros(shp) for _ in range(cfg.n_at)]
    V = [np.zeros(shp) for _ in range(cfg.n_at)]
    return OracleState(S, conv, K, V, 0, kv_q8)


# ------------------------------------------------------------------ the forward step
def _deltanet_mixer(cfg, W, p, st: OracleState, li: int, x: np.ndarray) -> np.ndarray:
    Hd, dk, dv = cfg.dn_heads, cfg.dn_dk, cfg.dn_dv
    C = cfg.dn_conv_channels
    z = W[p + "dn.w_in"] @ x                                   # [q; k; v; alpha; beta]
    raw, alpha, beta = z[:C], z[C:C + Hd], z[C + Hd:C + 2 * Hd]
    y = conv_silu(st.conv[li], raw, W[p + "dn.conv"])
    st.conv[li] = np.concatenate([st.conv[li][1:], raw[None, :]], axis=0)
    q = l2norm(y[:Hd * dk].reshape(Hd, dk))
    k = l2norm(y[Hd * dk:2 * Hd * dk].reshape(Hd, dk))
    v = y[2 * Hd * dk:].reshape(Hd, dv)
    a = np.exp(-softplus(alpha))
    b = sigmoid(beta)
    o = np.empty((Hd, dv))
    for h in range(Hd):
        st.S[li][h], o[h] = delta_rule_step(st.S[li][h], q[h], k[h], v[h], a[h], b[h])
    return o.reshape(-1)


def _attention_mixer(cfg, W, p, st: OracleState, li: int, x: np.ndarray) -> np.ndarray:
    Hq, Hkv, D = cfg.at_q_heads, cfg.at_kv_heads, cfg.at_head_dim
    z = W[p + "attn.w_in"] @ x                                 # [q; gate; k; v]
    off = 0
    q = z[off:off + Hq * D].reshape(Hq, D); off += Hq * D
    if cfg.at_out_gate:
        g = z[off:off + Hq * D]; off += Hq * D
    k = z[off:off + Hkv * D].reshape(Hkv, D); off += Hkv * D
    v = z[off:off + Hkv * D].reshape(Hkv, D)
    pos = st.pos
    q = rope(q, pos, cfg.rope_theta)
    k = rope(k, pos, cfg.rope_theta)
    if st.kv_q8:                              # 8-bit blocks of 32 with an fp16 scale
        st.K[li][:, pos] = q8_roundtrip(k)
        st.V[li][:, pos] = q8_roundtrip(v)
    else:                                     # the KV cache is stored in bf16
        st.K[li][:, pos] = round_bf16(k)
        st.V[li][:, pos] = round_bf16(v)
    o = attention_decode(q, st.K[li][:, :pos + 1], st.V[li][:, :pos + 1]).reshape(-1)
    if cfg.at_out_gate:
        o = o * sigmoid(g)
    return o


def decode_step(cfg, W, st: OracleState, tok: int, act_bf16: bool = False) -> np.ndarray:
    """Feed one token at position st.pos; returns the logits [vocab] and advances pos.

    The KV cache entries are always bf16 (stored state). act_bf16=True also rounds
    every projection input (normed hidden state, mixer output, SwiGLU activation)
    to bf16; by default they stay in full precision, as on the GPU, where they never
    leave the chip."""
    rnd = round_bf16 if act_bf16 else (lambda a: a)
    eps = cfg.rms_eps
    if st.K and st.pos >= st.K[0].shape[1]:
        raise ValueError("context capacity exceeded")
    h = W["embed"][int(tok)].copy()
    di = ai = 0
    for l, kind in enumerate(cfg.pattern):
        p = f"layers.{l}."
        x = rnd(rmsnorm(h, W[p + "norm1"], eps))
        if kind == "D":
            o = _deltanet_mixer(cfg, W, p, st, di, x); di += 1
            h = h + W[p + "dn.w_out"] @ rnd(o)
        else:
            o = _attention_mixer(cfg, W, p, st, ai, x); ai += 1
            h = h + W[p + "attn.w_out"] @ rnd(o)
        x = rnd(rmsnorm(h, W[p + "norm2"], eps))
        h = h + W[p + "mlp.w_down"] @ rnd(swiglu(x, W[p + "mlp.w_gate"], W[p + "mlp.w_up"]))
    x = rnd(rmsnorm(h, W["norm_f"], eps))
    st.pos += 1
    return W["embed"] @ x


def prefill(cfg, W, st: OracleState, tokens, act_bf16: bool = False) -> np.ndarray:
    """Feed a prompt token by token; returns the logits after the last one."""
    logits = None
    for t in tokens:
        logits = decode_step(cfg, W, st, int(t), act_bf16)
    return logits


def greedy_generate(cfg, W, st: OracleState, first_tok: int, n: int, act_bf16: bool = False,
                    keep_logits: bool = False):
    """Greedy decode of n tokens starting from first_tok (fed at st.pos).

    Returns (tokens[n], logits list or None): tokens[i] = argmax after feeding
    the i-th input, inputs being first_tok then tokens[:-1].
    """
    out, lg = [], []
    tok = int(first_tok)
    for _ in range(n):
        z = decode_step(cfg, W, st, tok, act_bf16)
        tok = int(np.argmax(z))          # first maximal index = lowest index on ties
        out.append(tok)
        if keep_logits:
            lg.append(z)
    return np.array(out, dtype=np.int32), (lg if keep_logits else None)


def verify_drafts(cfg, W, st: OracleState, last_tok: int, drafts, act_bf16: bool = False):
    """Speculative verify by its plain definition (exact greedy acceptance).

    Feeds [last_tok, d_1..d_K] one at a time on a copy of the state, recording
    g_i = argmax after the i-th input; n = the largest n with d_j = g_{j-1} for
    all j <= n. The committed tokens are d_1..d_n followed by the bonus g_n.
    The state is then rebuilt from the original by feeding [last_tok, d_1..d_n],
    so it ends exactly where plain greedy decoding of those tokens would.
    Returns (n_accepted, committed tokens[n+1], logits [K+1, V]).
    """
    drafts = [int(d) for d in drafts]
    trial = st.copy()
    feed = [int(last_tok)] + drafts
    g, logits = [], []
    for t in feed:
        z = decode_step(cfg, W, trial, t, act_bf16)
        logits.append(z)
        g.append(int(np.argmax(z)))
    n = 0
    while n < len(drafts) and drafts[n] == g[n]:
        n += 1
    committed = drafts[:n] + [g[n]]
    for t in feed[:n + 1]:
        decode_step(cfg, W, st, t, act_bf16)
    return n, np.array(committed, dtype=np.int32), np.stack(logits)
