"""Comparison metrics between the CUDA path and the oracle (test helpers)."""
import numpy as np

# Tolerances of the GPU path against the oracle.
LOGIT_MAX_ABS = 3e-2      # logits max-abs error
GREEDY_AGREE = 0.99       # teacher-forced greedy-token agreement
MEAN_KL = 1e-3            # mean KL(p_oracle || p_gpu), nats
STATE_REL_FROB = 1e-2     # DeltaNet state relative Frobenius error


def log_softmax(z):
    z = np.asarray(z, dtype=np.float64)
    m = z.max(axis=-1, keepdims=True)
    return z - m - np.log(np.exp(z - m).sum(axis=-1, keepdims=True))


def kl(z_ref, z_test):
    """KL(softmax(z_ref) || softmax(z_test)) per row, natural log."""
    lp = log_softmax(z_ref)
    lq = log_softmax(z_test)
    return (np.exp(lp) * (lp - lq)).sum(axis=-1)


def rel_frob(a, ref):
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-30))


def near_tie(z, margin=1e-2):
    s = np.sort(np.asarray(z))[::-1]
    return (s[0] - s[1]) < margin


def conv_history_as_window(ring, pos, width):
    """GPU conv history (slot p mod W holds position p) -> oracle window
    [W-1, C] of the last W-1 inputs, oldest first, after `pos` positions."""
    rows = []
    for m in range(width - 1, 0, -1):
        p = pos - m
        rows.append(ring[p % width] if p >= 0 else np.zeros_like(ring[0]))
    return np.stack(rows)


def assert_bf16_cache_close(got, want, rel_rms=5e-3, max_changed=0.15):
    """bf16 cache entries: both sides round a float value to bf16, so an entry may differ
    by one bf16 step when the two unrounded values straddle a rounding midpoint, and the
    unrounded values themselves differ by the path's activation error, which scales with
    the slice, not with a small entry. Bound per entry: one bf16 step at the larger of the
    two magnitudes plus rel_rms times the root mean square of its (layer, kv head) slice.
    At most max_changed of the entries may differ at all. A RoPE, ordering or position
    slip moves entries by about the slice's scale and fails the bound by orders of
    magnitude. On failure the message lists the worst entries (index, oracle, GPU) and the
    largest excess beyond one bf16 step, in units of the slice's RMS."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape
    lead = got.shape[:-2]
    g = got.reshape(-1, *got.shape[-2:])
    w = want.reshape(-1, *want.shape[-2:])
    for i in range(g.shape[0]):
        rms = float(np.sqrt(np.mean(w[i] ** 2))) if w[i].size else 0.0
        mag = np.maximum(np.abs(w[i]), np.abs(g[i]))
        ulp = np.where(mag > 0, 2.0 ** (np.floor(np.log2(np.maximum(mag, 1e-38))) - 7), 0.0)
        d = np.abs(g[i] - w[i])
        excess = np.maximum(d - ulp, 0.0) / max(rms, 1e-30)
        bad = excess > rel_rms
        if bad.any():
            order = np.argsort(excess, axis=None)[::-1][:5]
            worst = [(np.unravel_index(k, excess.shape), float(w[i].flat[k]), float(g[i].flat[k])) for k in order]
            raise AssertionError(f"slice {np.unravel_index(i, lead) if lead else i}: max excess "
                                 f"{float(excess.max()):.3g} x rms (rms {rms:.3g}); worst {worst}")
        assert (d > 0).mean() <= max_changed, float((d > 0).mean())
