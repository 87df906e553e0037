"""Seeded synthetic inputs shared by the library's checks and the oracle.
Holds none of the method's arithmetic."""
from .workloads import Workload, get, ALL, BY_INDEX, C0, C1, C2, C3, C4A, C4B  # noqa: F401
from .gradients import GradientSource, pack_offsets, mix_seed  # noqa: F401
