"""Plain, slow CPU oracle for MLA decoding over a paged latent KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code with
the CUDA library (``mla_paged_kv_get_b200``); the only thing both sides take is
the seeded input generator, which holds none of the method's arithmetic.

Modules
-------
``mla_oracle``  fp64 numpy restatement of the decode (dense two-pass and
                streaming/split forms) and of the split merge.
``schedule``    integer-only restatement of the tile scheduler that balances
                variable-length sequences over the SMs in page-sized pieces.
"""

from . import mla_oracle, schedule  # noqa: F401
