"""fp64 CPU oracle for the KDA recurrence.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product (``kimi_delta_attention_28_b200``) never imports it and shares no code
with it.
"""
from .kda_oracle import (kda_bwd, kda_bwd_packed, kda_decode_commit,  # noqa: F401
                         kda_decode_step, kda_decode_verify, kda_fwd, kda_fwd_packed,
                         threads_available)
