"""CPU oracle for group-wise affine weight quantization and the W4A16 matmul.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.
The CUDA library never calls it, and it shares no code with the CUDA library.
"""
from .wq_oracle import *  # noqa: F401,F403
