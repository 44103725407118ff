"""CPU oracle for the HXQ HelixLinear forward: test infrastructure only."""
from .hxq_oracle import *  # noqa: F401,F403
