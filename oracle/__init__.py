"""CPU oracle for NSA forward: TEST INFRASTRUCTURE, not part of the product.

Only the tests, the package smoke check and the bench's CPU-baseline leg may
import this package. The CUDA path never imports it and shares no code with it.
"""
from . import nsa_oracle, brute  # noqa: F401
