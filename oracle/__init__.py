"""Plain fp64 CPU oracle for 2D Neighborhood Attention.

Test infrastructure only: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it; the library never does.
"""
from .na2d_oracle import (  # noqa: F401
    build,
    forward,
    forward_points,
    forward_rows,
    qk_rpb,
    softmax,
    av,
    backward,
    sasa_forward,
    block_forward,
    nd_forward,
    window_start,
    max_threads,
)
