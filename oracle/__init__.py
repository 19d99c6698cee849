"""CPU oracle for PBSA (test infrastructure only; the library never imports it)."""
from .pbsa_oracle import *  # noqa: F401,F403
