"""fp64 CPU oracle for the Nystromformer attention forward pass.

Test infrastructure: only the tests, the smoke check and the benchmark's CPU
baseline leg use it.  The product path never imports it."""
from .nystrom import *  # noqa: F401,F403
