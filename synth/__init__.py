"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This module holds model shapes and random draws only. It holds none of the
model's arithmetic: no normalisation, projection, recurrence, attention or
dequantisation lives here. Both sides of every parity test take their inputs
from these functions and nothing else.

Random streams: every tensor is drawn from its own counter-based Philox-4x32-10
stream (Salmon et al., "Parallel random numbers: as easy as 1, 2, 3", SC 2011;
numpy's ``np.random.Philox``) keyed by ``(seed, fnv1a64(name))``, so a tensor's
values do not depend on which other tensors were generated or in what order.

Model shapes follow the hybrid layer pattern of the Hacker News post on the fused
24-layer Qwen3.5-0.8B kernel ("18 DeltaNet layers ... 6 Full Attention layers")
and the 27B-shaped engine of the open-jet megakernel follow-up post.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
from typing import Dict, List, Tuple

import numpy as np

# weight formats (mirrors MK_W_BF16 / MK_W_Q4K in the C header; plain ints)
W_BF16 = 0
W_Q4K = 1

Q4K_BLOCK = 256          # weights per super-block
Q4K_SUB = 32             # weights per sub-block (8 sub-blocks per super-block)
Q4K_BYTES = 144          # bytes per super-block: 2 fp16 + 12 B of 6-bit scales/mins + 128 B codes


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    name: str
    n_layers: int
    pattern: str              # one letter per layer: 'D' = Gated DeltaNet, 'A' = full attention
    hidden: int
    vocab: int
    rms_eps: float
    dn_heads: int
    dn_dk: int
    dn_dv: int
    conv_width: int
    at_q_heads: int
    at_kv_heads: int
    at_head_dim: int
    rope_theta: float
    at_out_gate: int          # 1: attention output is multiplied by sigmoid(gate rows)
    ffn: int
    weight_format: int = W_BF16
    seed: int = 0

    # ---- derived sizes (pure shape bookkeeping) ----
    @property
    def n_dn(self) -> int:
        return self.pattern.count("D")

    @property
    def n_at(self) -> int:
        return self.pattern.count("A")

    @property
    def dn_conv_channels(self) -> int:
        # the short conv runs over the q, k and v channels (not over alpha/beta)
        return self.dn_heads * (2 * self.dn_dk + self.dn_dv)

    @property
    def dn_in_rows(self) -> int:
        # [q; k; v; alpha; beta]
        return self.dn_conv_channels + 2 * self.dn_heads

    @property
    def at_in_rows(self) -> int:
        # [q; gate (if any); k; v]
        qd = self.at_q_heads * self.at_head_dim
        kvd = self.at_kv_heads * self.at_head_dim
        return qd * (2 if self.at_out_gate else 1) + 2 * kvd

    def param_count(self) -> int:
        n = self.vocab * self.hidden + self.hidden
        for kind in self.pattern:
            n += 2 * self.hidden + 3 * self.ffn * self.hidden
            if kind == "D":
                n += self.dn_in_rows * self.hidden + self.dn_conv_channels * self.conv_width
                n += self.hidden * self.dn_heads * self.dn_dv
            else:
                n += self.at_in_rows * self.hidden + self.hidden * self.at_q_heads * self.at_head_dim
        return n


def _preset(name: str, **kw) -> ModelConfig:
    return ModelConfig(name=name, **kw)


# The five workloads: a tiny CPU-check model, the 0.8B-shaped model (decode,
# prefill and long-context decode share it) and the 27B-shaped 4-bit model.
TINY = _preset("tiny", n_layers=4, pattern="DDDA", hidden=256, vocab=4096, rms_eps=1e-6,
               dn_heads=4, dn_dk=64, dn_dv=64, conv_width=4,
               at_q_heads=4, at_kv_heads=1, at_head_dim=64, rope_theta=1e7, at_out_gate=0,
               ffn=768, seed=0)
QWEN_08B = _preset("0.8b", n_layers=24, pattern="DDDA" * 6, hidden=1024, vocab=151936, rms_eps=1e-6,
                   dn_heads=16, dn_dk=128, dn_dv=128, conv_width=4,
                   at_q_heads=8, at_kv_heads=2, at_head_dim=256, rope_theta=1e7, at_out_gate=1,
                   ffn=3584, seed=1)
QWEN_27B = _preset("27b", n_layers=64, pattern="DDDA" * 16, hidden=5120, vocab=151936, rms_eps=1e-6,
                   dn_heads=48, dn_dk=128, dn_dv=128, conv_width=4,
                   at_q_heads=24, at_kv_heads=4, at_head_dim=256, rope_theta=1e7, at_out_gate=1,
                   ffn=17408, weight_format=W_Q4K, seed=4)
# A very small model with the same structure, for pure-Python cross-checks.
MINI = _preset("mini", n_layers=4, pattern="DDDA", hidden=32, vocab=64, rms_eps=1e-6,
               dn_heads=2, dn_dk=8, dn_dv=8, conv_width=4,
               at_q_heads=2, at_kv_heads=1, at_head_dim=8, rope_theta=1e7, at_out_gate=1,
               ffn=48, seed=7)

# 4-bit test shapes: the tiny model in the 4-bit format, and a mid-size model with the
# 27B model's head shapes (dk = dv = 128, gated attention) that the oracle runs in seconds.
TINY_Q4 = _preset("tiny-q4", n_layers=4, pattern="DDDA", hidden=256, vocab=4096, rms_eps=1e-6,
                  dn_heads=4, dn_dk=64, dn_dv=64, conv_width=4,
                  at_q_heads=4, at_kv_heads=1, at_head_dim=64, rope_theta=1e7, at_out_gate=0,
                  ffn=768, weight_format=W_Q4K, seed=10)
MID_Q4 = _preset("mid-q4", n_layers=8, pattern="DDDA" * 2, hidden=1024, vocab=32768, rms_eps=1e-6,
                 dn_heads=8, dn_dk=128, dn_dv=128, conv_width=4,
                 at_q_heads=8, at_kv_heads=2, at_head_dim=128, rope_theta=1e7, at_out_gate=1,
                 ffn=3072, weight_format=W_Q4K, seed=11)

# Four layers of the 27B shape (one [D,D,D,A] block): the 27B kernels on a small case
# (about 1.4 GB of 4-bit weights), for profiling.
QWEN_27B_4L = dataclasses.replace(QWEN_27B, name="27b-4l", n_layers=4, pattern="DDDA")

# The same four 27B-shaped layers with a 32K vocabulary: small enough for the float64 oracle
# (1.7 B weights), and it runs the hidden-5120 decode instance the 27B model runs.
QWEN_27B_4L_32K = dataclasses.replace(QWEN_27B, name="27b-4l-32k", n_layers=4, pattern="DDDA", vocab=32768)

# Two models whose decode scratch leaves no room for the whole layer table, so the decode
# kernel keeps two table slots and fetches each layer's entry during the layer before (as
# the 64-layer 27B model does): eight query heads of 256 per KV head need 5656 floats of
# attention scratch per CTA, and the bf16 hidden size of 2880, or the 4-bit FFN of 16640
# (staged whole by the down-projection), takes the room that eight table entries would need.
WIDE_GQA8 = _preset("wide-gqa8", n_layers=8, pattern="DDDA" * 2, hidden=2880, vocab=4096, rms_eps=1e-6,
                    dn_heads=4, dn_dk=128, dn_dv=128, conv_width=4,
                    at_q_heads=8, at_kv_heads=1, at_head_dim=256, rope_theta=1e7, at_out_gate=1,
                    ffn=1024, seed=12)
WIDE_GQA8_Q4 = _preset("wide-gqa8-q4", n_layers=8, pattern="DDDA" * 2, hidden=256, vocab=4096, rms_eps=1e-6,
                       dn_heads=4, dn_dk=128, dn_dv=128, conv_width=4,
                       at_q_heads=8, at_kv_heads=1, at_head_dim=256, rope_theta=1e7, at_out_gate=1,
                       ffn=16640, weight_format=W_Q4K, seed=13)

CONFIGS = {c.name: c for c in (TINY, QWEN_08B, QWEN_27B, MINI, TINY_Q4, MID_Q4, QWEN_27B_4L, QWEN_27B_4L_32K,
                               WIDE_GQA8, WIDE_GQA8_Q4)}


def with_changes(cfg: ModelConfig, **kw) -> ModelConfig:
    return dataclasses.replace(cfg, **kw)


# ---------------------------------------------------------------- random streams
def _fnv1a64(s: str) -> int:
    h = 0xCBF29CE484222325
    for ch in s.encode():
        h ^= ch
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def stream(seed: int, name: str) -> np.random.Generator:
    """Independent Philox stream for (seed, name)."""
    key = np.array([seed & 0xFFFFFFFFFFFFFFFF, _fnv1a64(name)], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Storage encoding of the synthetic weights: fp32 -> bf16 bit pattern,
    round to nearest, ties to even (finite inputs only)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    u = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Storage decoding: bf16 bit pattern -> fp32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------- tensor specs
def tensor_specs(cfg: ModelConfig) -> List[Tuple[str, Tuple[int, ...], str]]:
    """(name, shape, init) for every weight tensor, in load order.

    init: 'normal' = N(0, 0.02); 'gain' = 1 + N(0, 0.02) (RMSNorm gains);
    'conv' = N(0, 0.02) with the current-token tap (last column) + 1.
    Linear weights are [out_features, in_features] (row-major).
    """
    H = cfg.hidden
    specs = [("embed", (cfg.vocab, H), "normal")]
    for l, kind in enumerate(cfg.pattern):
        p = f"layers.{l}."
        specs.append((p + "norm1", (H,), "gain"))
        if kind == "D":
            specs.append((p + "dn.w_in", (cfg.dn_in_rows, H), "normal"))
            specs.append((p + "dn.conv", (cfg.dn_conv_channels, cfg.conv_width), "conv"))
            specs.append((p + "dn.w_out", (H, cfg.dn_heads * cfg.dn_dv), "normal"))
        else:
            specs.append((p + "attn.w_in", (cfg.at_in_rows, H), "normal"))
            specs.append((p + "attn.w_out", (H, cfg.at_q_heads * cfg.at_head_dim), "normal"))
        specs.append((p + "norm2", (H,), "gain"))
        specs.append((p + "mlp.w_gate", (cfg.ffn, H), "normal"))
        specs.append((p + "mlp.w_up", (cfg.ffn, H), "normal"))
        specs.append((p + "mlp.w_down", (H, cfg.ffn), "normal"))
    specs.append(("norm_f", (H,), "gain"))
    return specs


def is_quantized(cfg: ModelConfig, name: str, shape) -> bool:
    """Under the 4-bit format every 2-D projection (the tied embedding included)
    is stored as Q4_K-style blocks; conv taps and RMSNorm gains stay bf16."""
    return cfg.weight_format == W_Q4K and len(shape) == 2 and not name.endswith("dn.conv")


def _draw_f32(cfg: ModelConfig, seed: int, name: str, shape, init: str) -> np.ndarray:
    g = stream(seed, name)
    x = g.standard_normal(int(np.prod(shape)), dtype=np.float32).reshape(shape)
    x *= np.float32(0.02)
    if init == "gain":
        x += np.float32(1.0)
    elif init == "conv":
        x[:, -1] += np.float32(1.0)
    return x


def make_weights(cfg: ModelConfig, seed: int | None = None, threads: int = 8) -> Dict[str, np.ndarray]:
    """All weights of ``cfg`` as raw storage arrays.

    bf16 tensors come back as uint16 bit patterns with the tensor's shape.
    Under the 4-bit format, quantised tensors come back as uint8 arrays of
    shape [rows, cols // 256 * 144] (see ``quantize_q4k``).
    """
    seed = cfg.seed if seed is None else seed
    specs = tensor_specs(cfg)

    def one(spec):
        name, shape, init = spec
        x = _draw_f32(cfg, seed, name, shape, init)
        if is_quantized(cfg, name, shape):
            return name, quantize_q4k(x)
        return name, f32_to_bf16_bits(x)

    with _cf.ThreadPoolExecutor(max(1, threads)) as ex:
        return dict(ex.map(one, specs))


# ---------------------------------------------------------------- Q4_K-style encoding
def quantize_q4k(w: np.ndarray) -> np.ndarray:
    """Encode fp32 weights [rows, cols] (cols % 256 == 0) into 144-byte super-blocks.

    This is how the synthetic 4-bit model is *made*; the model is the codes.
    Per 32-weight sub-block j: lo = min(min(w), 0), hi = max(w); scale_j = (hi - lo)/15,
    min_j = -lo. Per super-block: d = max_j scale_j / 63, dmin = max_j min_j / 63 (fp16);
    sc_j = round(scale_j / d), m_j = round(min_j / dmin) in [0, 63];
    q = clamp(round((w + dmin*m_j) / (d*sc_j)), 0, 15). Rounding is half-to-even.

    Byte layout of one super-block (little endian):
      [0:2]  d    (fp16)      [2:4] dmin (fp16)
      [4:16] 16 six-bit fields, LSB-first bit stream: sc_0..sc_7 then m_0..m_7
      [16:144] codes: sub-block j occupies bytes 16+16j .. 16+16j+15; byte t holds
               q[32j + t] in its low nibble and q[32j + t + 16] in its high nibble.
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    assert cols % Q4K_BLOCK == 0
    nb = cols // Q4K_BLOCK
    x = w.reshape(rows, nb, 8, Q4K_SUB).astype(np.float64)
    lo = np.minimum(x.min(axis=3), 0.0)
    hi = x.max(axis=3)
    scale = (hi - lo) / 15.0
    mn = -lo
    d = (scale.max(axis=2) / 63.0).astype(np.float16)
    dmin = (mn.max(axis=2) / 63.0).astype(np.float16)
    d64 = d.astype(np.float64)[..., None]
    dm64 = dmin.astype(np.float64)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        sc = np.where(d64 > 0, np.rint(scale / np.where(d64 > 0, d64, 1.0)), 0.0)
        m = np.where(dm64 > 0, np.rint(mn / np.where(dm64 > 0, dm64, 1.0)), 0.0)
    sc = np.clip(sc, 0, 63).astype(np.int64)
    m = np.clip(m, 0, 63).astype(np.int64)
    step = d64 * sc                                  # [rows, nb, 8]
    off = dm64 * m
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(step[..., None] > 0,
                     np.rint((x + off[..., None]) / np.where(step[..., None] > 0, step[..., None], 1.0)),
                     0.0)
    q = np.clip(q, 0, 15).astype(np.uint8)          # [rows, nb, 8, 32]

    out = np.zeros((rows, nb, Q4K_BYTES), dtype=np.uint8)
    out[:, :, 0:2] = d.view(np.uint8).reshape(rows, nb, 2)
    out[:, :, 2:4] = dmin.view(np.uint8).reshape(rows, nb, 2)
    # 16 six-bit fields -> 96-bit little-endian stream -> 12 bytes
    fields = np.concatenate([sc, m], axis=2).astype(np.uint64)   # [rows, nb, 16]
    lo64 = np.zeros((rows, nb), dtype=np.uint64)
    hi64 = np.zeros((rows, nb), dtype=np.uint64)
    for f in range(16):
        bit = 6 * f
        v = fields[:, :, f]
        if bit + 6 <= 64:
            lo64 |= v << np.uint64(bit)
        elif bit >= 64:
            hi64 |= v << np.uint64(bit - 64)
        else:                                        # straddles the 64-bit boundary
            lo64 |= (v << np.uint64(bit)) & np.uint64(0xFFFFFFFFFFFFFFFF)
            hi64 |= v >> np.uint64(64 - bit)
    for bpos in range(8):
        out[:, :, 4 + bpos] = ((lo64 >> np.uint64(8 * bpos)) & np.uint64(0xFF)).astype(np.uint8)
    for bpos in range(4):
        out[:, :, 12 + bpos] = ((hi64 >> np.uint64(8 * bpos)) & np.uint64(0xFF)).astype(np.uint8)
    lo_n = q[..., :16]
    hi_n = q[..., 16:]
    codes = (lo_n | (hi_n << 4)).astype(np.uint8)   # [rows, nb, 8, 16]
    out[:, :, 16:] = codes.reshape(rows, nb, 128)
    return out.reshape(rows, nb * Q4K_BYTES)


# ---------------------------------------------------------------- token streams
def make_prompt(cfg: ModelConfig, n: int, seed: int | None = None, tag: str = "prompt") -> np.ndarray:
    """n uniform token ids in [0, vocab)."""
    seed = cfg.seed if seed is None else seed
    return stream(seed, tag).integers(0, cfg.vocab, size=n, dtype=np.int64).astype(np.int32)


def draft_choices(seed: int, pass_idx: int, k: int, vocab: int, p_greedy: float = 0.8):
    """Per draft slot: (use_greedy: bool[k], random ids int32[k]).

    The caller turns them into drafts: slot i takes the greedy token when
    use_greedy[i], else the random id, redrawn upward (id+1 mod vocab) while it
    equals the greedy token.
    """
    g = stream(seed, f"drafts.{pass_idx}")
    use = g.random(k) < p_greedy
    ids = g.integers(0, vocab, size=k, dtype=np.int64).astype(np.int32)
    return use, ids


def compose_drafts(greedy: np.ndarray, use: np.ndarray, ids: np.ndarray, vocab: int) -> np.ndarray:
    out = np.where(use, greedy, ids).astype(np.int32)
    for i in range(len(out)):
        if not use[i]:
            while out[i] == greedy[i]:
                out[i] = (out[i] + 1) % vocab
    return out


# ---------------------------------------------------------------- long-context state
def long_context_state(cfg: ModelConfig, n_pos: int, seed: int = 3):
    """Seeded long-context state: per attention layer K, V of shape [Hkv, n_pos, D]
    (bf16 bit patterns) and per DeltaNet layer S of shape [Hd, dv, dk] (fp32).

    K and V are i.i.d. N(0, 1). Keys are stored as already rotated: a rotation
    of an isotropic Gaussian pair is again isotropic Gaussian, so drawing the
    rotated keys directly has the same distribution as drawing then rotating.
    S entries are i.i.d. N(0, 0.1); conv tails start at zero.
    """
    shp = (cfg.at_kv_heads, n_pos, cfg.at_head_dim)
    ks, vs, ss = [], [], []
    for i in range(cfg.n_at):
        ks.append(f32_to_bf16_bits(stream(seed, f"kv.k.{i}").standard_normal(shp, dtype=np.float32)))
        vs.append(f32_to_bf16_bits(stream(seed, f"kv.v.{i}").standard_normal(shp, dtype=np.float32)))
    for i in range(cfg.n_dn):
        s = stream(seed, f"state.S.{i}").standard_normal((cfg.dn_heads, cfg.dn_dv, cfg.dn_dk), dtype=np.float32)
        ss.append((s * np.float32(0.1)).astype(np.float32))
    return ks, vs, ss


# ---------------------------------------------------------------- device-side 4-bit blocks
def device_q4_weights(cfg: ModelConfig, dev, seed: int):
    """Weights of the 4-bit model for timing: every Q4 super-block generated on the device
    (uniform codes and 6-bit fields, fp16 d and dmin in [2^-15, 2^-14)), gains and conv taps
    from the seeded stream. Parity at these head shapes is tested on the mid-size 4-bit model;
    this only sizes the work (14.4 GB of 4-bit weights)."""
    import torch
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    out = {}
    for name, shape, init in tensor_specs(cfg):
        if is_quantized(cfg, name, shape):
            rows, cols = shape
            nb = cols // 256
            t = torch.randint(0, 256, (rows, nb, 144), dtype=torch.uint8, device=dev, generator=g)
            dd = ((torch.rand((rows, nb, 2), device=dev, generator=g) + 1.0) * 2.0 ** -15).to(torch.float16)
            t[:, :, 0:4] = dd.view(torch.uint8).reshape(rows, nb, 4)
            out[name] = t.reshape(rows, nb * 144)
        else:
            x = _draw_f32(cfg, seed, name, shape, init)
            out[name] = torch.from_numpy(f32_to_bf16_bits(x).view(np.int16)).to(dev).view(torch.bfloat16)
    return out
