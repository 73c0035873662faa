"""CPU oracle for head-split attention (test infrastructure only)."""
from .duo_oracle import *  # noqa: F401,F403
