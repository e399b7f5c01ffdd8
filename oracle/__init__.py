"""Float64 CPU oracle (test infrastructure only; see ``gqa_ref``)."""
from .gqa_ref import *  # noqa: F401,F403
