"""fp64 CPU oracle for the RMM hot path. Test infrastructure only: the library
never imports it, and it imports nothing from the library."""
from .rmm_oracle import *  # noqa: F401,F403
