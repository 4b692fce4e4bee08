"""Float64 CPU oracle for block-hybrid attention.  Test infrastructure only: imported by
the test suite, the package smoke check and the bench's CPU-baseline leg, never by the
library itself."""
from .bha_ref import *  # noqa: F401,F403
