"""CPU oracle for the hybrid Gated-DeltaNet + attention forward step.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or
link this package: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

It is the plain definition of what the CUDA path computes, written in numpy
with float64 arithmetic, token by token (the recurrent form), with one
library primitive per step (matrix-vector products, a triangular solve).
It shares no code with the CUDA path; both read their inputs from ``synth``.

Rounding contract: weights are bf16 and the KV cache entries are stored in bf16;
every other quantity stays in full precision (float64 here, float32 on the GPU,
where activations live in registers and shared memory and never leave the chip).
``act_bf16=True`` additionally rounds every projection input (normalised hidden
state, mixer output, SwiGLU activation) to bf16 -- the megakernel post's bf16
activations taken literally -- for diagnostics.
"""
from .model import *          # noqa: F401,F403
from .chunked import *        # noqa: F401,F403
from .q4k import *            # noqa: F401,F403
from .sampling import *       # noqa: F401,F403
from .kvq8 import *           # noqa: F401,F403
from .sequence import *       # noqa: F401,F403
