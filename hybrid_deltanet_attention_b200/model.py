"""Thin Python binding over libmk.so: argument marshalling only.

PyTorch provides device memory (the packed weights, the state and the workspace
are torch uint8 tensors) and streams; every step of the forward pass runs in the
library's kernels.
"""
from __future__ import annotations

import ctypes as C
from typing import Dict, Optional

import numpy as np
import torch

from . import _abi
from ._abi import MkConfig, MkSizes, MkTensor, check


def make_config(cfg, max_ctx: int, max_draft: int = 0, kv_format: int = 0) -> MkConfig:
    """Build the C config from any object with the model-shape attributes
    (n_layers, pattern, hidden, vocab, rms_eps, dn_heads, dn_dk, dn_dv, conv_width,
    at_q_heads, at_kv_heads, at_head_dim, rope_theta, at_out_gate, ffn, weight_format)."""
    c = MkConfig()
    c.n_layers = cfg.n_layers
    c.pattern = cfg.pattern.encode()
    c.hidden = cfg.hidden
    c.vocab = cfg.vocab
    c.rms_eps = cfg.rms_eps
    c.dn_heads = cfg.dn_heads
    c.dn_dk = cfg.dn_dk
    c.dn_dv = cfg.dn_dv
    c.conv_width = cfg.conv_width
    c.at_q_heads = cfg.at_q_heads
    c.at_kv_heads = cfg.at_kv_heads
    c.at_head_dim = cfg.at_head_dim
    c.rope_theta = cfg.rope_theta
    c.at_out_gate = cfg.at_out_gate
    c.ffn = cfg.ffn
    c.weight_format = cfg.weight_format
    c.max_ctx = max_ctx
    c.max_draft = max_draft
    c.kv_format = kv_format
    return c


def query_sizes(cfg, max_ctx: int, max_draft: int = 0, kv_format: int = 0) -> MkSizes:
    """mk_query_sizes for a model shape on the current CUDA device: buffer sizes, state
    offsets, the decode grid and the decode kernel's layer-table form."""
    sizes = MkSizes()
    check(_abi.load_library().mk_query_sizes(C.byref(make_config(cfg, max_ctx, max_draft, kv_format)),
                                             C.byref(sizes)))
    return sizes


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


class Model:
    """One model instance on the current CUDA device.

    weights: name -> CUDA tensor (torch.bfloat16, or torch.uint16/int16 bf16 bit
    patterns). They are repacked into the model's own buffer; the caller may drop
    them after construction.
    """

    def __init__(self, cfg, weights: Dict[str, torch.Tensor], max_ctx: int, max_draft: int = 0,
                 stream: Optional[torch.cuda.Stream] = None, kv_format: int = 0):
        self.lib = _abi.load_library()
        self.shape = cfg
        self.kv_format = int(kv_format)
        self.cfg = make_config(cfg, max_ctx, max_draft, self.kv_format)
        self.sizes = MkSizes()
        check(self.lib.mk_query_sizes(C.byref(self.cfg), C.byref(self.sizes)))
        dev = torch.device("cuda", torch.cuda.current_device())
        sz = self.sizes
        self.packed = torch.empty(int(sz.packed_bytes), dtype=torch.uint8, device=dev)
        self.state = torch.empty(int(sz.state_bytes), dtype=torch.uint8, device=dev)
        self.workspace = torch.empty(int(sz.workspace_bytes), dtype=torch.uint8, device=dev)
        arr = (MkTensor * len(weights))()
        self._names = []
        for i, (name, t) in enumerate(weights.items()):
            if not t.is_cuda:
                raise ValueError(f"weight {name} must be a CUDA tensor")
            t = t.contiguous()
            nb = name.encode()
            self._names.append(nb)
            arr[i].name = nb
            if t.dtype in (torch.bfloat16, torch.int16, torch.uint16):
                arr[i].dtype = _abi.MK_DT_BF16
            elif t.dtype == torch.uint8:
                arr[i].dtype = _abi.MK_DT_Q4K
            elif t.dtype == torch.float32:
                arr[i].dtype = _abi.MK_DT_F32
            else:
                arr[i].dtype = 0
            arr[i].ndim = t.dim()
            for d in range(min(4, t.dim())):
                arr[i].shape[d] = t.shape[d]
            if arr[i].dtype == _abi.MK_DT_Q4K and t.dim() == 2:
                arr[i].shape[1] = t.shape[1] // 144 * 256     # logical columns of the 144-byte super-blocks
            arr[i].data = t.data_ptr()
            arr[i].bytes = t.numel() * t.element_size()
        handle = C.c_void_p()
        check(self.lib.mk_load_weights(C.byref(self.cfg), arr, len(weights), self.packed.data_ptr(),
                                       self.state.data_ptr(), self.workspace.data_ptr(), _stream_ptr(stream),
                                       C.byref(handle)))
        self.h = handle
        self._tok = torch.zeros(8, dtype=torch.int32, device=dev)

    def __del__(self):
        h = getattr(self, "h", None)
        if h is not None and h.value:
            self.lib.mk_free(h)
            self.h = None

    # ---- state views (documented layout of the state buffer) ----
    def _view(self, off: int, dtype, shape):
        n = int(np.prod(shape))
        esz = torch.tensor([], dtype=dtype).element_size()
        return self.state[off:off + n * esz].view(dtype).view(*shape)

    @property
    def S(self) -> torch.Tensor:
        c = self.shape
        return self._view(self.sizes.off_S, torch.float32, (c.n_dn, c.dn_heads, c.dn_dv, c.dn_dk))

    @property
    def conv_history(self) -> torch.Tensor:
        c = self.shape
        return self._view(self.sizes.off_conv, torch.float32, (c.n_dn, c.conv_width, c.dn_conv_channels))

    def _kv_view(self, off: int) -> torch.Tensor:
        c = self.shape
        if self.kv_format == _abi.MK_KV_Q8:      # raw rows: D int8 codes, D/32 fp16 scales, padding
            return self._view(off, torch.uint8, (c.n_at, c.at_kv_heads, self.cfg.max_ctx, int(self.sizes.kv_row_bytes)))
        return self._view(off, torch.bfloat16, (c.n_at, c.at_kv_heads, self.cfg.max_ctx, c.at_head_dim))

    @property
    def k_cache(self) -> torch.Tensor:
        return self._kv_view(self.sizes.off_k)

    @property
    def v_cache(self) -> torch.Tensor:
        return self._kv_view(self.sizes.off_v)

    def kv_q8_rows(self, which: str):
        """8-bit cache rows split into (codes int8 [n_at, Hkv, max_ctx, D], scales float16
        [n_at, Hkv, max_ctx, D/32]), on the host."""
        D = self.shape.at_head_dim
        raw = (self.k_cache if which == "k" else self.v_cache).cpu()
        codes = raw[..., :D].contiguous().view(torch.int8)
        scales = raw[..., D:D + D // 16].contiguous().view(torch.float16)
        return codes.numpy(), scales.numpy()

    @property
    def pos_tensor(self) -> torch.Tensor:
        return self._view(self.sizes.off_pos, torch.int32, (1,))

    # ---- calls ----
    def reset(self, stream=None):
        check(self.lib.mk_reset_state(self.h, _stream_ptr(stream)))

    def set_position(self, pos: int, stream=None):
        check(self.lib.mk_set_position(self.h, int(pos), _stream_ptr(stream)))

    def prefill(self, tokens: torch.Tensor, logits: Optional[torch.Tensor] = None,
                next_token: Optional[torch.Tensor] = None, stream=None):
        assert tokens.dtype == torch.int32 and tokens.is_cuda
        check(self.lib.mk_prefill(self.h, tokens.data_ptr(), tokens.numel(), _ptr(logits), _ptr(next_token),
                                  _stream_ptr(stream)))

    def decode(self, in_token: torch.Tensor, out_token: torch.Tensor, logits: Optional[torch.Tensor] = None,
               stream=None):
        check(self.lib.mk_decode_step(self.h, in_token.data_ptr(), out_token.data_ptr(), _ptr(logits),
                                      _stream_ptr(stream)))

    def verify(self, tokens: torch.Tensor, n_accepted: torch.Tensor, out_tokens: torch.Tensor,
               logits: Optional[torch.Tensor] = None, stream=None):
        K = tokens.numel() - 1
        check(self.lib.mk_verify_drafts(self.h, tokens.data_ptr(), K, n_accepted.data_ptr(), out_tokens.data_ptr(),
                                        _ptr(logits), _stream_ptr(stream)))

    def verify_sampled(self, tokens: torch.Tensor, temperature: float, uniforms: torch.Tensor,
                       n_accepted: torch.Tensor, out_tokens: torch.Tensor, logits: Optional[torch.Tensor] = None,
                       stream=None):
        """Sampling-mode verify; uniforms: float32 CUDA tensor of 2 * tokens.numel() values in [0, 1)."""
        K = tokens.numel() - 1
        assert uniforms.dtype == torch.float32 and uniforms.is_cuda and uniforms.numel() >= 2 * (K + 1)
        check(self.lib.mk_verify_drafts_sampled(self.h, tokens.data_ptr(), K, float(temperature),
                                                uniforms.data_ptr(), n_accepted.data_ptr(), out_tokens.data_ptr(),
                                                _ptr(logits), _stream_ptr(stream)))

    def generate(self, prompt, n_new: int, stream=None, out: Optional[np.ndarray] = None) -> np.ndarray:
        """Host prompt in, host tokens out (pinned or pageable numpy int32 arrays)."""
        p = np.ascontiguousarray(prompt, dtype=np.int32)
        o = out if out is not None else np.empty(n_new, dtype=np.int32)
        check(self.lib.mk_generate(self.h, p.ctypes.data, p.size, o.ctypes.data, n_new, _stream_ptr(stream)))
        return o

    def sync(self, stream=None) -> int:
        err = C.c_int32(0)
        rc = self.lib.mk_sync_status(self.h, _stream_ptr(stream), C.byref(err))
        if rc != _abi.MK_OK:
            raise _abi.MkError(rc, (self.lib.mk_last_error() or b"").decode() + f" (device word 0x{err.value:x})")
        return err.value

    def device_error(self) -> int:
        err = C.c_int32(0)
        self.lib.mk_sync_status(self.h, _stream_ptr(None), C.byref(err))
        return err.value

    def phase_trace(self, buf: Optional[torch.Tensor]):
        """Diagnostics: record per-barrier timestamps of CTA 0 into buf (int64 CUDA tensor), or stop (None)."""
        if buf is None:
            check(self.lib.mk_phase_trace(self.h, None, 0))
        else:
            check(self.lib.mk_phase_trace(self.h, buf.data_ptr(), buf.numel()))

    @property
    def launches(self) -> int:
        return int(self.lib.mk_launch_count(self.h))


def weights_to_device(raw: Dict[str, np.ndarray], device="cuda") -> Dict[str, torch.Tensor]:
    """Storage arrays (bf16 bit patterns as uint16, Q4 bytes as uint8) -> CUDA tensors."""
    out = {}
    for k, v in raw.items():
        if v.dtype == np.uint16:
            out[k] = torch.from_numpy(v.view(np.int16)).to(device).view(torch.bfloat16)
        else:
            out[k] = torch.from_numpy(v).to(device)
    return out
