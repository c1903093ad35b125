"""CPU oracle for the GPT-OSS Mixture-of-Experts FFN layer -- TEST INFRASTRUCTURE.

This package is the plain, slow, obviously-correct statement of what the layer
computes.  It exists to check the CUDA library, and nothing on the product path
may import, call or link it: only the tests, the smoke check and the benchmark's
CPU-baseline leg use it.  It shares no code, table or constant with the CUDA
path; both sides only consume the same seeded inputs (``workloads``).

Two levels:
  * ``moe_oracle`` (O1): numpy, fp64 arithmetic on the exact input values,
    per-expert matmuls through numpy's BLAS;
  * ``brute``      (O0): pure-Python scalar loops, for tiny inputs only; it is
    what O1 is pinned against.

``glm_moe`` is the O1 oracle of the layer's GLM4-MoE-Lite variant (sigmoid
router with a selection-only correction bias, SiLU experts, a shared expert);
``mx_act`` the O1 oracle of the MXFP4 layer with its activations in MXFP8 (the
block-scaled numerics variant); ``brute`` holds the scalar-loop counterparts of
both.

Every function is pinned by ``tests/test_oracle_pins*.py`` (brute force, closed
forms, invariants, hand-worked values in ``tests/golden/``).  No function here
is "parity unpinned".
"""
from . import moe_oracle, brute, glm_moe, mx_act  # noqa: F401
