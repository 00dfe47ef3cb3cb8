"""FP64 CPU oracle for the fused LM-head projection + cross-entropy.

Test infrastructure only: the product path never imports this package.
"""
from .flce_oracle import *  # noqa: F401,F403
