"""fp64 CPU oracle (test infrastructure only; never on the product path)."""
from .oracle import Oracle, compile_library, default  # noqa: F401
