"""fp64 CPU oracle (test infrastructure only; never on the product path).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It shares no code with the CUDA path.
"""
from .attention import (  # noqa: F401
    NEG_INF,
    allowed_keys,
    attention_keyset,
    attention_reference,
    attention_rows,
    block_allowed,
    kv_head,
    merge_partials,
    ring_attention_online,
    shard_tokens,
    softmax_row,
)
from .backward import (  # noqa: F401
    attention_backward_reference,
    backward_rows_dkdv,
    backward_rows_dq,
    delta_rows,
    ring_attention_backward_online,
)
from .decode import decode_reference, decode_split  # noqa: F401
