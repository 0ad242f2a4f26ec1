"""Float64 CPU oracle for the pack -> attend -> unpack path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()`` and by the
CPU-baseline leg of ``bench.py``; never by the product package.  It shares no code with the
CUDA path.
"""
from .oracle import (  # noqa: F401
    build,
    cu_seqlens,
    rank,
    pack,
    attend,
    attend_rows,
    unpack,
    library_path,
    l2_mask,
    l2_score,
)
