"""Float64 CPU oracle for the POET-X layer.  Test infrastructure only (see poetx_ref)."""
from . import poetx_ref  # noqa: F401
