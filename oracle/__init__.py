"""Float64 CPU oracle of the CSA / HCA hot path. TEST INFRASTRUCTURE: imported only by
the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg; never by the
product library or its binding."""
from . import csa_oracle, pipeline, state_cache  # noqa: F401
