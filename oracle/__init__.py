"""CPU oracle of the rotated low-bit linear layer: test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU-baseline leg use this
package.  The product path (the CUDA library and its binding) never imports it.
"""
from .rbd_oracle import *  # noqa: F401,F403
