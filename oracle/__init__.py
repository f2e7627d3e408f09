"""Float64 CPU oracle for TwoTower block attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The CUDA library never does.
"""
from .oracle import attend_rows, block_attn, block_causal  # noqa: F401
from .brute import brute_block_attn, brute_block_causal  # noqa: F401
from .kv_append import kv_append  # noqa: F401
from .backward import block_causal_backward  # noqa: F401
from .unmask import confidence_unmask  # noqa: F401
from .paged import block_attn_paged, gather_pages  # noqa: F401
