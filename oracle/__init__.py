"""fp64 CPU oracle for retrieval block-sparse attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the library calls this package: only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
import it.  It shares no code with the CUDA path; both read the same seeded
inputs from ``retrieval_block_sparse_b200.synth`` and nothing else.

Every function is pinned against closed forms, invariants, library routines
or brute force: ``tests/test_oracle_pins.py`` (retrieval attention),
``tests/test_oracle_memory_pins.py`` (dynamic memory update) and
``tests/test_oracle_approx_pins.py`` (two-stage approximate retrieval) and
``tests/test_oracle_gated_pins.py`` (landmark-gated attention); see
the docstring of each function for the passage of the pages it restates.
"""
from .retrieval import *  # noqa: F401,F403
from .retrieval import __all__ as _r_all
from .memory import *  # noqa: F401,F403
from .memory import __all__ as _m_all
from .approx import *  # noqa: F401,F403
from .approx import __all__ as _a_all
from .gated import *  # noqa: F401,F403
from .gated import __all__ as _g_all

__all__ = list(_r_all) + list(_m_all) + list(_a_all) + list(_g_all)
