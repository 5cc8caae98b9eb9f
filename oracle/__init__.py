"""CPU oracle for the expert-parallel MoE-layer forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path (the
C-ABI library and its Python binding) never imports, links or calls it, and the
oracle never imports the product package: the two share no code.  The only
module both sides use is ``moe_workloads`` (seeded input draws, no arithmetic).

Every function is a plain restatement of the method's definition in float64
numpy, citing the page and section it follows.  See ``moe_oracle`` for the
functions and the readings taken where the pages are silent.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import __all__  # noqa: F401
