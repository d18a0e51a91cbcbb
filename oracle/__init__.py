"""CPU oracle for SageSLA attention: test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package. It shares no code with the CUDA path.
"""
from .sagesla_oracle import (  # noqa: F401
    BLOCK, Prepared, Selection, block_logits, block_means, channel_mean, counts, fma32,
    forward, linear_states, phi, prepare, quantize_blocks, round_bf16, sagesla, select,
    softmax_scale,
)
