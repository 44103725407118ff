"""CPU oracle for the HXQ HelixLinear forward and encoder: test infrastructure only."""
from .hxq_encoder_oracle import *  # noqa: F401,F403
from .hxq_oracle import *  # noqa: F401,F403
