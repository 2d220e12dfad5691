"""fp64 CPU oracle of windowed RIB attention + CLA gate (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg import this package. The product path (``windowed_attention_b200``)
never imports it and shares no code with it.
"""
from .rib_oracle import *  # noqa: F401,F403
