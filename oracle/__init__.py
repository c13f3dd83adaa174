"""CPU oracle for the BitLinear hot path (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
legs may import this package. It shares no code with bit_ternary_b200.
"""
from .bitlinear_oracle import *  # noqa: F401,F403
from .bitlinear_oracle import __all__ as _core_all
from .i2s_oracle import *  # noqa: F401,F403
from .i2s_oracle import __all__ as _i2s_all
from .block_oracle import *  # noqa: F401,F403
from .block_oracle import __all__ as _block_all

__all__ = list(_core_all) + list(_i2s_all) + list(_block_all)
