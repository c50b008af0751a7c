"""CPU oracle of the MoE token shuffle (route -> dispatch -> grouped SwiGLU FFN -> combine).

TEST INFRASTRUCTURE ONLY: plain, slow, obviously correct restatements of what the path computes.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs may
import this package.  It shares no code with the CUDA library and never reads its outputs.
"""
from . import moe, numerics  # noqa: F401
