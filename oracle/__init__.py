"""fp64 CPU oracle (test infrastructure only; see svg_oracle.py and svg2_oracle.py)."""
from .svg_oracle import *  # noqa: F401,F403
from .svg2_oracle import *  # noqa: F401,F403
