"""CPU oracle for the quantized MoE expert-gather path.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this package; only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may call it.  It shares no code with the CUDA path (``csrc/``), and the CUDA path
never falls back to it.

Everything here is plain numpy, written to be checked against the pages by eye:
fp32 where the method fixes fp32 (quantisation and dequantisation), fp64 for every
matmul, activation and sum.  See ``qmoe_oracle`` for the per-function citations.

Parity status of each function (what pins it, in ``tests/test_oracle_*.py``):

* ``bf16_from_f32`` / ``f32_from_bf16``   pinned: hand-computed bit patterns.
* ``pack_codes`` / ``unpack_codes``       pinned: hand-computed words for 1-8-bit codes
                                          (straddling 3/5/6-bit codes included), round trip.
* ``quantize`` / ``dequantize``           pinned: the error bounds and constructed
                                          groups of nuvec-core's quantized.rs tests over
                                          every width it tests, hand-worked groups.
* ``qmm`` / ``gather_qmm``                pinned: exact rational arithmetic
                                          (``fractions``) on tiny shapes, per-batch
                                          selection identity, sorted == unsorted.
* ``sort_by_expert`` / ``tile_table``     pinned: MLX PR #4567's worked example,
                                          brute-force enumeration.
* ``switch_glu``                          pinned: closed forms on hand-built weights.
* ``moe_combine``                         pinned: reduction to a plain unsort, a
                                          mean, and closed-form gates.

No function is "parity unpinned".
"""

from .qmoe_oracle import *  # noqa: F401,F403
