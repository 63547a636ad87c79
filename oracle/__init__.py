"""CPU oracle for the tensor-parallel MLP / attention block (fp64 numpy).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA path never imports, links or calls anything in here, and this
package imports nothing from the CUDA path.

See ``oracle/tp_oracle.py`` for the functions and the passages they follow.
"""
from .tp_oracle import *  # noqa: F401,F403
