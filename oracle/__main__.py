"""`python -m oracle [--force]` compiles the oracle library (test infrastructure)."""
import sys

from . import build

print(build(force="--force" in sys.argv))
