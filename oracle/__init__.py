"""fp64 CPU oracle for the fused attention forward.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / ``--impl reference`` legs, never by the
library. It shares no code with the CUDA path.
"""
from .attention import *  # noqa: F401,F403
from .attention import (attention_rows, attention_varlen, attention_padded, attention_paged,
                        combine, decode, mla_paged, mla_sparse, mla_sparse_tnd, visible_mask,
                        visible_range,
                        gather_pages)
