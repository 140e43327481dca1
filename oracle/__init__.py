"""Oracle for the gated-delta-rule token mixer -- test infrastructure only.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg may
import this package.  The product path (the CUDA library and its binding) never
imports, links or calls anything here; the two share no code.
"""
from .gdn_oracle import (  # noqa: F401
    build,
    conv,
    gated_rmsnorm,
    gates,
    l2norm,
    mixer,
    num_threads,
    recurrence,
)
from .chunked import chunked_recurrence, chunked_transfer_recurrence  # noqa: F401
from .projections import gemm, in_proj_layout, layer, round_bf16  # noqa: F401
from . import attention as attn  # noqa: F401
