"""fp64 CPU oracle (test infrastructure; never imported by the product path)."""
from . import isloss_oracle  # noqa: F401
from . import model_oracle  # noqa: F401
