"""A second, independently written float64 forward step in plain Python.

Used only to cross-check the numpy oracle on a very small model. It uses
Python lists, ``math`` and ``struct`` only: no numpy, no code from ``oracle``.
Per token: embed -> for each layer (pre-norm mixer, residual; pre-norm SwiGLU,
residual) -> final norm -> tied LM head.
"""
import math
import struct


def bf16(x):
    """Round a Python float to the nearest bf16 value (ties to even) via fp32 bits."""
    (u,) = struct.unpack("<I", struct.pack("<f", x))
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFFFFFF
    (f,) = struct.unpack("<f", struct.pack("<I", (u >> 16) << 16))
    return f


def from_bits(b):
    """bf16 bit pattern (int) -> Python float."""
    (f,) = struct.unpack("<f", struct.pack("<I", (int(b) & 0xFFFF) << 16))
    return f


def decode(arr):
    """Nested list of bf16 bit patterns (numpy uint16 array) -> nested list of floats."""
    lst = arr.tolist()
    if isinstance(lst[0], list):
        return [[from_bits(v) for v in row] for row in lst]
    return [from_bits(v) for v in lst]


def matvec(W, x):
    return [math.fsum(w * xi for w, xi in zip(row, x)) for row in W]


def rms(h, g, eps):
    s = math.sqrt(math.fsum(v * v for v in h) / len(h) + eps)
    return [h[i] / s * g[i] for i in range(len(h))]


def sig(x):
    return 1.0 / (1.0 + math.exp(-x))


class PyModel:
    def __init__(self, cfg, raw):
        """raw: dict name -> bf16 bit-pattern array, as produced by ``synth.make_weights``."""
        self.c = cfg
        self.W = {k: decode(v) for k, v in raw.items()}
        c = cfg
        self.S = [[[[0.0] * c.dn_dk for _ in range(c.dn_dv)] for _ in range(c.dn_heads)]
                  for _ in range(c.n_dn)]
        self.hist = [[[0.0] * c.dn_conv_channels for _ in range(c.conv_width - 1)] for _ in range(c.n_dn)]
        self.K = [[] for _ in range(c.n_at)]
        self.V = [[] for _ in range(c.n_at)]
        self.pos = 0

    def step(self, tok, act=False):
        """act=True also rounds every projection input to bf16; the KV cache is always bf16."""
        c, W = self.c, self.W
        r = bf16 if act else (lambda v: v)
        h = list(W["embed"][tok])
        di = ai = 0
        for l, kind in enumerate(c.pattern):
            p = "layers.%d." % l
            x = [r(v) for v in rms(h, W[p + "norm1"], c.rms_eps)]
            if kind == "D":
                o = self._dn(p, di, x)
                di += 1
                h = [a + b for a, b in zip(h, matvec(W[p + "dn.w_out"], [r(v) for v in o]))]
            else:
                o = self._at(p, ai, x)
                ai += 1
                h = [a + b for a, b in zip(h, matvec(W[p + "attn.w_out"], [r(v) for v in o]))]
            x = [r(v) for v in rms(h, W[p + "norm2"], c.rms_eps)]
            gt = matvec(W[p + "mlp.w_gate"], x)
            up = matvec(W[p + "mlp.w_up"], x)
            act = [r(g * sig(g) * u) for g, u in zip(gt, up)]
            h = [a + b for a, b in zip(h, matvec(W[p + "mlp.w_down"], act))]
        x = [r(v) for v in rms(h, W["norm_f"], c.rms_eps)]
        self.pos += 1
        return matvec(W["embed"], x)

    def _dn(self, p, li, x):
        c, W = self.c, self.W
        Hd, dk, dv, Cw = c.dn_heads, c.dn_dk, c.dn_dv, c.conv_width
        C = c.dn_conv_channels
        z = matvec(W[p + "dn.w_in"], x)
        raw = z[:C]
        taps = W[p + "dn.conv"]
        hist = self.hist[li]
        y = []
        for ch in range(C):
            seq = [hist[j][ch] for j in range(Cw - 1)] + [raw[ch]]
            s = math.fsum(taps[ch][j] * seq[j] for j in range(Cw))
            y.append(s * sig(s))
        self.hist[li] = hist[1:] + [raw]
        out = []
        for hd in range(Hd):
            q = y[hd * dk:(hd + 1) * dk]
            k = y[Hd * dk + hd * dk:Hd * dk + (hd + 1) * dk]
            v = y[2 * Hd * dk + hd * dv:2 * Hd * dk + (hd + 1) * dv]
            nq = math.sqrt(math.fsum(t * t for t in q) + 1e-6)
            nk = math.sqrt(math.fsum(t * t for t in k) + 1e-6)
            q = [t / nq for t in q]
            k = [t / nk for t in k]
            al = z[C + hd]
            be = z[C + Hd + hd]
            a = sig(-al)                      # exp(-softplus(al)) == sigmoid(-al)
            b = sig(be)
            S = self.S[li][hd]
            for i in range(dv):
                row = [a * t for t in S[i]]
                u = math.fsum(row[j] * k[j] for j in range(dk))
                S[i] = [row[j] + b * (v[i] - u) * k[j] for j in range(dk)]
            out += [math.fsum(S[i][j] * q[j] for j in range(dk)) for i in range(dv)]
        return out

    def _at(self, p, li, x):
        c, W = self.c, self.W
        Hq, Hkv, D = c.at_q_heads, c.at_kv_heads, c.at_head_dim
        z = matvec(W[p + "attn.w_in"], x)
        q = z[:Hq * D]
        off = Hq * D
        g = None
        if c.at_out_gate:
            g = z[off:off + Hq * D]
            off += Hq * D
        k = z[off:off + Hkv * D]
        v = z[off + Hkv * D:off + 2 * Hkv * D]

        def rot(vec, pos):
            half = D // 2
            o = list(vec)
            for i in range(half):
                ang = pos * c.rope_theta ** (-2.0 * i / D)
                cs, sn = math.cos(ang), math.sin(ang)
                o[i] = vec[i] * cs - vec[i + half] * sn
                o[i + half] = vec[i] * sn + vec[i + half] * cs
            return o

        qs = [rot(q[h * D:(h + 1) * D], self.pos) for h in range(Hq)]
        ks = [[bf16(t) for t in rot(k[h * D:(h + 1) * D], self.pos)] for h in range(Hkv)]
        vs = [[bf16(t) for t in v[h * D:(h + 1) * D]] for h in range(Hkv)]
        self.K[li].append(ks)
        self.V[li].append(vs)
        out = []
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            sc = [math.fsum(qs[h][d] * self.K[li][j][kv][d] for d in range(D)) / math.sqrt(D)
                  for j in range(self.pos + 1)]
            m = max(sc)
            e = [math.exp(t - m) for t in sc]
            zz = math.fsum(e)
            o = [math.fsum(e[j] * self.V[li][j][kv][d] for j in range(len(e))) / zz for d in range(D)]
            if g is not None:
                o = [o[d] * sig(g[h * D + d]) for d in range(D)]
            out += o
        return out
