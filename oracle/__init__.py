"""Float64 CPU oracle (test infrastructure only; never a fallback for the CUDA path)."""
from . import cag64, hsa64  # noqa: F401
