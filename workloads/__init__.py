"""Named workloads and their seeded synthetic inputs (no method arithmetic)."""
from .configs import ALL, BY_NAME, MEM_100M, MEM_16M, MEM_16M_B32, MEM_1M, TINY_F32, Workload  # noqa: F401
from . import gen  # noqa: F401
