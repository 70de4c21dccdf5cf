"""CPU oracle for FP8 per-tensor quantization and per-tensor-scaled FP8 GEMM.

TEST INFRASTRUCTURE ONLY. This package is the plain, slow, obviously correct
reference that the CUDA path is checked against. Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. The product library never imports,
links or calls anything here, and nothing here imports the product library:
the two share no code, no tables and no constants generators.

Method (what is computed), after the AstrAI FP8 commit logs:

* ``astrai/extension/fp8.py @4dc5e923`` -- the delayed-scaling ring: the
  quantize step folds the tensor's amax into ``hist[idx]``, reduces the
  window and publishes the next scale; the amax is taken over the
  *unquantized* values (the fix for the scale that collapsed to 1).
* ``astrai/extension/fp8.py @f4c44ebf`` -- the GEMM dequantizes with the
  scale the quantize actually used (snapshot before the ring finalize); the
  bias is added in fp32 before the single bf16 rounding; 3-D operands with
  stride-0 broadcast; bf16 is the only GEMM output type.
* ``tests/extension/test_fp8_mma.py @cebdd45d`` -- a null ``bias_scale``
  means a raw bf16 bias, a non-null one means fp8 bias storage dequantized
  after the operand scaling.

Where the pages are silent the OCP 8-bit floating point specification
(OFP8, rev. 1.0) fixes the formats, and the readings listed in each module
header fix the rest.

Precision: codec and quantize follow the fp32 arithmetic the method fixes
(the product x*scale is formed exactly in fp64 and rounded once to fp32);
the GEMM accumulates in fp64 and rounds once from fp64 to bf16.

Parity pins: every function here is pinned in ``tests/test_oracle_*.py``
against facts that do not come from this code (OFP8 boundary values, an
independent library cast, exact rational brute force, hand-computed ring
tables). One reading is **parity unpinned**: the treatment of NaN inputs in
the amax (NaN is ignored), which the pages do not fix; no configuration
contains NaN. The GPU tests hold the kernel to this reading on every bf16
pattern, NaNs included.
"""

from .codec import (  # noqa: F401
    E4M3,
    E5M2,
    FMT_MAX,
    decode,
    decode_table,
    encode,
    bf16_round_from_f64,
    bf16_bits_to_f32,
)
from .quantize import (  # noqa: F401
    amax,
    current_scale,
    quantize_with_scale,
    quantize_current,
    DelayedRing,
    HISTORY,
)
from .gemm import (  # noqa: F401
    NT,
    NN,
    TN,
    mm,
    mm_exact,
    mm_out8,
    mm_sampled,
    tolerance,
    fp8_ulp,
    out8_tolerance,
)
from .linear import (  # noqa: F401
    bias_grad,
    bias_grad_tolerance,
    Fp8LinearRef,
)
