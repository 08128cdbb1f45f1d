"""fp64 CPU oracle of the MoVA value path.  Test infrastructure only: the
tests, the smoke check and the benchmark's CPU-baseline leg may use it; the
CUDA library never does."""
from .mova_oracle import *  # noqa: F401,F403
