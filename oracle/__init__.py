"""Plain CPU float64 oracle for the TurboQuant KV-cache hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library (``kv_cache_vector_11_b200``); the two meet only on the seeded
synthetic inputs from ``workloads``.

Every step follows the method as the source pages describe it and is written
for readability, not speed: dense matrices, numpy float64, one formula per
line.  Where the pages leave a step open the docstring says which reading is
taken.  Sources (page title, then section):

* "TurboQuant+ upstream guide: llama.cpp KV cache compression, 4-phase PR
  roadmap" (bjdmk.com.cn) -- section 3 (Codex finding 6: seeded rotation
  generation, QR -> Haar, slogdet for det=+1), section 4 (dense rotation vs the
  D1 @ H @ D2 Walsh-Hadamard rotation), section 5.1 (MSE-only PolarQuant,
  block 32, per-block norm extraction and rescale), section 5.2 (block
  struct, centroid table), section 5.3 (pre-rotated queries,
  <q, R^T c[idx]> = <R q, c[idx]>; asymmetric K/V; inverse-rotation fix).
* "Plan de Integracion: TurboQuant en Orion" (stig.sh) -- "Implementacion
  conceptual": QJL keeps one sign bit per projected residual value.
* "Google TurboQuant deep dive" (lonae.com) -- section 2.2 (QJL: random
  Gaussian projection of the residual, then sign binarisation; the query
  stays full precision), section 4.2 (JL lemma), section 4.3
  (softmax(Q K^T / sqrt(d)) V).

Parity status: every public function is pinned by ``tests/test_oracle_*.py``
to closed forms, invariants, textbook values, brute force or an independent
library routine.  None is "parity unpinned".
"""

from . import rng, rotation, codebook, quant, qjl, attention, search, paged  # noqa: F401
