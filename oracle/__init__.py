"""CPU oracle for the hybrid Gated-DeltaNet + attention forward step.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or
link this package: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

It is the plain definition of what the CUDA path computes, written in numpy
with float64 arithmetic, token by token (the recurrent form), with one
library primitive per step (matrix-vector products, a triangular solve).
It shares no code with the CUDA path; both read their inputs from ``synth``.

Rounding contract (the megakernel post's "BF16 weights and activations, FP32
accumulation"): weights are bf16; the vectors that feed a projection (the
normalised hidden state, the mixer output, the SwiGLU activation) and the KV
cache entries are rounded to bf16; everything else stays in full precision
(float64 here, float32 on the GPU). ``round_inputs=False`` drops the bf16
rounding of activations for diagnostics.
"""
from .model import *          # noqa: F401,F403
from .chunked import *        # noqa: F401,F403
from .q4k import *            # noqa: F401,F403
