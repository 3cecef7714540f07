"""CPU oracle for the looped-block hot path.  TEST INFRASTRUCTURE ONLY: the
product library never imports it; tests, the smoke check and the benchmark's
CPU-baseline leg do."""
from .tinyloop_oracle import *  # noqa: F401,F403
from .workloads import build_oracle_model, packed_weights  # noqa: F401
