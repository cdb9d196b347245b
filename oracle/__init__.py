"""fp64 CPU oracle of the routed MoE layer forward -- test infrastructure.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  It shares no code with the CUDA
library and never receives a value computed by it.
"""

from .moe_oracle import *  # noqa: F401,F403
from .eplb_oracle import *  # noqa: F401,F403
from .dedup_oracle import *  # noqa: F401,F403
from .fp8_oracle import *  # noqa: F401,F403
from .ep_oracle import *  # noqa: F401,F403
from . import dedup_oracle as _dedup
from . import ep_oracle as _ep
from . import eplb_oracle as _eplb
from . import fp8_oracle as _fp8
from . import moe_oracle as _moe

__all__ = (list(_moe.__all__) + list(_eplb.__all__) + list(_dedup.__all__)
           + list(_fp8.__all__) + list(_ep.__all__))
