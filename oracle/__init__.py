"""CPU oracle of one FreeToken-style MoE layer forward pass with an expert cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It shares
no code with the CUDA library (``expert_offloaded_serving_b200``) and imports
nothing from it; the two meet only through the seeded inputs of ``synth``.

Plain, slow and fp64 throughout, written from the public write-ups of FreeToken
(cited per function) plus the readings stated where those pages are silent:

* ``fp4``      e2m1 / UE8M0 decoding, the scale-atom storage index, the OCP MX
               quantiser and fp64 -> bf16 rounding.
* ``routing``  fixed-order router logits, softmax top-k, stable permutation.
* ``layer``    SwiGLU expert FFN and the weighted combine (decode bf16 mode and
               MXFP4-activation mode).
* ``lru``      the global LRU expert cache across layers, with resize.
* ``formats``  BF16 and NVFP4 expert blobs (decode only), decoded to fp64.
* ``cpp``      the same functions from ``ft_oracle.cpp``, a plain C++17
               restatement (built by ``oracle/build.py`` into liboracle.so,
               OpenMP over the experts of a layer for the timed CPU baseline).
               The numpy modules are its cross-check (tests/test_oracle_cpp.py).

Pins (tests/test_oracle_*.py, all CPU): exhaustive code x scale tables against
the closed form, hand-computed scale-atom offsets, quantiser ties and
idempotence, brute-force top-k with injected ties, stable-sort permutation
invariants, a hand-computed two-expert layer (tests/golden/), the partition
invariant of the combine, an LRU checked against a timestamp simulation, and
sign, idempotence and quantised-input invariants of the quantiser and of the
MXFP4 expert.  tests/test_oracle_mutants.py plants 44 plausible mistakes in
this package one at a time (wrong table entries, nibble and byte orders,
rounding and tie rules, summation orders, swapped operands, dropped terms,
recency rules); each makes at least one of those pins fail.
No function here is "parity unpinned".
"""
from . import fp4, formats, routing, layer, lru  # noqa: F401
# ``oracle.cpp`` is imported on use: it compiles liboracle.so on first load
