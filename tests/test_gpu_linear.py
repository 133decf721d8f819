"""The tensor-core linear layer (mk_linear) through the C ABI against a float64 product.

X is fp32, W bf16. The kernel multiplies W by X's bf16 high and low parts into one fp32
accumulator, which keeps about 16 bits of X's mantissa; the bound below allows
2^-15 of sum |x||w| per output plus the fp32 accumulation.
"""
import ctypes as C

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _bf16_matrix(rng, n, k, scale=0.02):
    bits = synth.f32_to_bf16_bits(rng.standard_normal((n, k), dtype=np.float32) * np.float32(scale))
    vals = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return bits, vals


def _run(M, N, K, accumulate=False, row_pad_bytes=0, seed=0):
    import hybrid_deltanet_attention_b200 as hda
    lib = hda.load_library()
    rng = np.random.default_rng(seed)
    dev = torch.device("cuda")
    bits, w = _bf16_matrix(rng, N, K)
    ldw = 2 * K + row_pad_bytes
    wbuf = np.zeros((N, ldw), dtype=np.uint8)
    wbuf[:, :2 * K] = bits.view(np.uint8).reshape(N, 2 * K)
    x = rng.standard_normal((M, K), dtype=np.float32)
    c0 = rng.standard_normal((M, N), dtype=np.float32) if accumulate else np.zeros((M, N), np.float32)
    d_w = torch.from_numpy(wbuf).to(dev)
    d_x = torch.from_numpy(x).to(dev)
    d_c = torch.from_numpy(c0.copy()).to(dev)
    scratch = torch.empty(max(16, 4 * M * K), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.mk_linear(d_x.data_ptr(), K, M, K, d_w.data_ptr(), ldw, N, d_c.data_ptr(), N, int(accumulate),
                       scratch.data_ptr(), scratch.numel(), err.data_ptr(), C.c_void_p(stream))
    assert rc == 0, lib.mk_last_error()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = d_c.cpu().numpy().astype(np.float64)
    want = x.astype(np.float64) @ w.T + c0.astype(np.float64)
    bound = 2.0 ** -15 * (np.abs(x).astype(np.float64) @ np.abs(w).T) + 1e-6 + 2e-7 * np.abs(c0)
    assert np.all(np.abs(got - want) <= bound), float(np.max(np.abs(got - want) / bound))
    return got


@pytest.mark.parametrize("M,N,K", [(1, 64, 64), (37, 200, 256), (128, 128, 128), (300, 1000, 512)])
def test_linear_ragged_shapes(M, N, K):
    _run(M, N, K)


def test_linear_accumulate_into_c():
    _run(130, 300, 256, accumulate=True, seed=3)


def test_linear_padded_weight_rows_and_wide_tile():
    # DeltaNet in-projection rows carry a 16-byte tail; N >= 2048 takes the 256-wide tile
    _run(520, 2304, 1024, row_pad_bytes=16, seed=5)


def test_linear_rejects_bad_sizes():
    import hybrid_deltanet_attention_b200 as hda
    lib = hda.load_library()
    dev = torch.device("cuda")
    buf = torch.zeros(1 << 16, dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    p = buf.data_ptr()
    # K not a multiple of 64
    assert lib.mk_linear(p, 96, 4, 96, p, 192, 4, p, 4, 0, p, buf.numel(), err.data_ptr(), None) == -1
    # scratch too small
    assert lib.mk_linear(p, 64, 64, 64, p, 128, 4, p, 4, 0, p, 100, err.data_ptr(), None) == -1


@pytest.mark.parametrize("M,N,K,seed", [(4096, 6176, 1024, 7), (2048, 7168, 1024, 8), (4096, 1024, 3584, 9)])
def test_linear_many_tiles_per_cta(M, N, K, seed):
    """Hundreds of output tiles (800, 448 and 128-plus-K-split work items at the prefill's
    in-projection, gate/up and down shapes): each persistent CTA walks several tiles and
    alternates its two TMEM accumulators, so one tile's epilogue overlaps the next tile's
    MMAs. Every element is checked against the float64 product."""
    _run(M, N, K, row_pad_bytes=16 if N == 6176 else 0, seed=seed)
