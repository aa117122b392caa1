"""CPU oracle (test infrastructure only; see ``s5_oracle``)."""
from .s5_oracle import *  # noqa: F401,F403
from . import s5_oracle  # noqa: F401
