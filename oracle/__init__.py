"""CPU oracle of the LCP hot path (test infrastructure; see lcp_oracle's header)."""
from . import lcp_oracle  # noqa: F401
