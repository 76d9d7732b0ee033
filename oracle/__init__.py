"""CPU oracle for the SVDQuant W4A4 + low-rank linear layer (test infrastructure only)."""
from .oracle import *  # noqa: F401,F403
from .oracle import build, lib  # noqa: F401
