"""CPU oracle (test infrastructure only; see ``oracle.paged_attention``, ``oracle.tree_accept``, ``oracle.fp8``,
``oracle.prefix_cache`` and ``oracle.lookahead_cache``)."""
from .paged_attention import (  # noqa: F401
    gather_sequence_kv,
    paged_kv_append,
    paged_tree_attention,
    softmax_attend,
    visible_positions,
    widen_to_f64,
    within_tolerance,
)
from . import tree_accept  # noqa: F401,E402
from . import fp8  # noqa: F401,E402
from . import prefix_cache  # noqa: F401,E402
from . import lookahead_cache  # noqa: F401,E402
