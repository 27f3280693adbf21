"""CPU oracle (test infrastructure only; see w4a16_oracle's header)."""
from .w4a16_oracle import *  # noqa: F401,F403
from .w4a16_oracle import ASYM, SYM, SLOT_TO_ELEM  # noqa: F401
