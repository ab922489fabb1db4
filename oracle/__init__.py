"""CPU oracle for the decode LM-head / projection GEMV path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the C-ABI library, the
Python binding, the kernels) imports, links or calls this package; only the
test-suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
legs of ``bench.py`` do.  It shares no code, table or helper with the CUDA
sources under ``decode_lm_head_b200/csrc``.

Everything here is a plain, slow restatement of the method in float64 numpy,
with the formats decoded from their definitions:

* ``numerics``  - E4M3 / E2M1 / E8M0 / BF16 / F16 decode and encode.
* ``gemv``      - the hot-path operations (FP8 W8A16, W8A8 quantize + GEMV,
                  fused SiLU quantize, NVFP4 W4A16, q8_1 quantize, Q6_K x q8_1).
* ``plan``      - the row-chunk and tier rules of the host dispatch.

Pinning status (what each function is checked against, in ``tests/``):
pinned by library routines, closed forms, printed tables and brute force.  The
element order inside a Q6_K super-block, which the pages do not print, is pinned
by hand-derived single-byte probes and by the gguf library's Q6_K dequantizer
(see ``gemv.q6k_unpack``).
"""

from . import numerics, gemv, plan  # noqa: F401
