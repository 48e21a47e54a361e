"""fp64 CPU oracle for the tensor-parallel layers: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path
(``linear_layers_b200``) never imports it, and the two share no code: the
only module both sides use is ``tp_inputs``, which draws seeded random
inputs and holds none of the layers' arithmetic.
"""
from .tp_oracle import *  # noqa: F401,F403
from .tp_oracle import (ACT_GELU_ERF, ACT_GELU_TANH, ACT_NONE, act_fwd,  # noqa: F401
                        act_grad, all_reduce_sum, even_offsets)
