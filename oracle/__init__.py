"""fp64 CPU oracle for the Veda tile-skipping attention layer (test
infrastructure: imported only by the tests, the smoke check and the
benchmark's CPU-baseline leg; never by the library)."""
from . import veda_oracle  # noqa: F401
