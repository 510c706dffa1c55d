"""Plain fp64 CPU oracle of the Lighthouse Attention hot path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import, call or execute
anything in this package. The product path (``long_context_symmetric_b200``)
never imports it, and this package imports nothing from the CUDA side: the two
share no code, tables, constants or helpers.

Everything here is written from the method's description in
"Long Context Pre-Training with Lighthouse Attention" (Peng, Ghosh, Quesnelle;
arXiv 2605.06554) and the summaries of it; see the header of
``oracle/lighthouse.py`` for the sources and the readings taken where the
description is silent.
"""

from .lighthouse import *  # noqa: F401,F403
from . import sharded  # noqa: F401,E402
