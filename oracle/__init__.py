"""CPU oracle of the DSA layer group (test infrastructure only; see dsa_oracle).

Only tests, the smoke check and the bench's CPU-baseline leg may import this package.
The product path never does: it runs only the CUDA library.
"""
from .dsa_oracle import *  # noqa: F401,F403
