"""Seeded synthetic inputs shared by the tests, the bench and the oracle legs."""

from .synthetic import (BUILDERS, WORKLOAD_NAMES, Workload, keys_at, make_workload,  # noqa: F401
                        prefill_inputs, slots_of)
from .projections import ProjectionWeights, make_projections  # noqa: F401
