"""fp64 CPU oracle for the KV-bank hot path.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import,
call or execute anything in this package.  The CUDA library never routes through
it, and it shares no code, header, table or constant generator with the library.

Each function restates, in plain and slow NumPy fp64, what one step of the method
computes, following the two pages that define it:

* DensityKV -- "DensityKV: Density-Guided KV Cache Compression for Long Video
  Generation" (summary page: §3 Method, App. A.1, App. B.1 "Online Bank Update",
  App. D, App. E; abstract page: Fig. 2).
* Forcing-KV -- "Forcing-KV: Hybrid KV Cache Compression for Efficient
  Autoregressive Video Diffusion Models" (reading notes: §3.3 static structural
  pruning, §3.4 dynamic similarity pruning, §3.5 code map).

Where the pages name a quantity without its formula, the oracle takes one plain
reading; every such reading is listed in the module that uses it.
Pins: see ``tests/test_oracle_*.py``.  Parity with the real DensityKV paper's
(unpublished on the pages) Soft-Riesz formula is unpinned; the reading below is.
"""
from .density import soft_riesz, sq_dists, density  # noqa: F401
from .attention import attention  # noqa: F401
from . import densitykv, forcingkv  # noqa: F401
