"""fp64 CPU oracle for the ODA / DA decode path. Test infrastructure only: imported by the
tests, the smoke check and the bench's CPU-baseline leg, never by the product path."""
from .oda_oracle import *  # noqa: F401,F403
