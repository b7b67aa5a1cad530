"""fp64 CPU oracle of the Muon / NorMuon step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline
may import this package; the CUDA library never does.
"""
from .muon_oracle import *  # noqa: F401,F403
from .muon_oracle import __all__ as _core_all
from .polar_express import *  # noqa: F401,F403
from .polar_express import __all__ as _pe_all

__all__ = list(_core_all) + list(_pe_all)
