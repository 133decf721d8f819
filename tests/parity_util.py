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
