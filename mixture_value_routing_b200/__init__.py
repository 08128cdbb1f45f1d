"""MoVA value path on NVIDIA B200: a C-ABI CUDA library (libmova.so) and its
thin Python binding (``mixture_value_routing_b200.api``).  See include/mova.h
for the ABI."""
from ._lib import LIB_PATH, MovaError  # noqa: F401
