"""CPU oracle for the BitLinear hot path (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
legs may import this package. It shares no code with bit_ternary_b200.
"""
from .bitlinear_oracle import *  # noqa: F401,F403
from .bitlinear_oracle import __all__  # noqa: F401
