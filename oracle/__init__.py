"""CPU oracle for the TurboQuant KV-cache codec and decode attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (the CUDA library and its Python binding) never
imports, links or runs anything here, and nothing here imports the product.
"""
from .tq_oracle import *  # noqa: F401,F403
