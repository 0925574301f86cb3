"""CPU oracle for the H-BitLinear forward pass.

Test infrastructure only: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path.
"""
from .hbl_oracle import *  # noqa: F401,F403
from .hbl_oracle import __all__  # noqa: F401
