"""fp64 CPU oracle for split-value-cache attention.

Test infrastructure: only the tests, ``__graft_entry__.smoke()`` and the bench's
CPU-baseline leg may import it.  It shares no code with the CUDA library.
"""

from .lrkv_oracle import *  # noqa: F401,F403
from .lrkv_oracle import BASE_SHARED, BASE_LR_SHARED  # noqa: F401
