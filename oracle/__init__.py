"""Float64 CPU oracle (test infrastructure only; never a fallback for the CUDA path)."""
from . import hsa64  # noqa: F401
