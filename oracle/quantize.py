"""Per-tensor FP8 quantization: amax, current scaling and the delayed ring.

Test infrastructure only (see the package docstring).

What the AstrAI commit logs fix:

* amax is the maximum magnitude of the *unquantized* input; measuring it on
  the quantized values (always about 448) made the scale collapse to 1
  (``astrai/extension/fp8.py @4dc5e923``, bullets on the amax bug; the
  ``@f4c44ebf`` page's tests use fp32-domain amax references).
* delayed scaling keeps a history ring; the quantize step writes the new
  amax into ``hist[idx]``, reduces the window and publishes the next scale,
  all after quantizing (``astrai/extension/fp8.py @4dc5e923``, bullet on the
  last-block epilogue).
* the GEMM must dequantize with the scale the quantize used, captured before
  the finalize overwrites it (``astrai/extension/fp8.py @f4c44ebf``, bullet
  on the sx/sw/sg snapshot) -- hence ``step`` returns the scale it used.
* dynamic ("current") scaling uses no ring and measures the scale from the
  tensor itself (``astrai/extension/fp8.py @4dc5e923``, bullet on the
  dynamic-scaling path).

Readings taken where the pages are silent:

* scale is the multiplier into FP8: q = sat_rne(fp32(x * scale)); the
  product is one IEEE fp32 rounding of the exact product, then one FP8
  rounding (never through fp16).
* scale = fmt_max / amax in IEEE fp32 division, with no margin and no
  power-of-two rounding; a quotient that overflows fp32 is clamped to the
  largest finite fp32 value.
* current scaling with amax = 0 or a non-finite amax uses scale 1.
* a seeded ring call quantizes with the current scale of its input and then
  folds that amax as usual (``DelayedRing.seed_step``).
* the ring holds H = 16 entries, starts at hist = 0, idx = 0, scale = 1.
* a window maximum that is 0 or non-finite keeps the previous scale.
* the window includes the amax just written.
* NaN inputs are ignored by the amax (**parity unpinned** for this one
  reading: the pages fix no NaN behaviour and no configuration contains NaN;
  the amax itself is pinned on finite inputs, and the GPU kernel is compared
  with this reading on every bf16 pattern, NaNs included).
"""

import numpy as np

from .codec import FMT_MAX, encode

HISTORY = 16
_FLT_MAX = np.float32(np.finfo(np.float32).max)


def amax(x) -> np.float32:
    """max |x| over fp32 values (bf16 inputs widen exactly); 0 if empty."""
    x = np.asarray(x, dtype=np.float32).reshape(-1)
    if x.size == 0:
        return np.float32(0.0)
    m = np.nanmax(np.abs(x)) if not np.all(np.isnan(x)) else np.float32(0.0)
    return np.float32(m)


def _fmax_over(fmt: int, a: np.float32) -> np.float32:
    """fp32(fmt_max / a), clamped to the largest finite fp32 value.

    fp64 division of two fp32 operands followed by one rounding to fp32
    equals the correctly rounded fp32 quotient (53 >= 2*24 + 2, so the double
    rounding is harmless for division).
    """
    with np.errstate(over="ignore"):
        q = np.float32(np.float64(FMT_MAX[fmt]) / np.float64(a))
    return _FLT_MAX if np.isinf(q) else q


def current_scale(a, fmt: int) -> np.float32:
    """Scale of dynamic ("current") scaling from the tensor's own amax."""
    a = np.float32(a)
    if a > 0 and np.isfinite(a):
        return _fmax_over(fmt, a)
    return np.float32(1.0)


def quantize_with_scale(x, scale, fmt: int) -> np.ndarray:
    """FP8 codes of fp32(x * scale); x holds bf16 values as fp32."""
    x = np.asarray(x, dtype=np.float32)
    # the product of two fp32 values is exact in fp64; one rounding to fp32
    p = (x.astype(np.float64) * np.float64(np.float32(scale))).astype(np.float32)
    return encode(p, fmt)


def quantize_current(x, fmt: int):
    """Current scaling: returns (codes, amax, scale used)."""
    a = amax(x)
    s = current_scale(a, fmt)
    return quantize_with_scale(x, s, fmt), a, s


class DelayedRing:
    """Delayed-scaling amax history of one tensor role (H = 16)."""

    def __init__(self, init_scale: float = 1.0):
        self.hist = np.zeros(HISTORY, dtype=np.float32)
        self.idx = 0
        self.scale = np.float32(init_scale)

    def copy(self) -> "DelayedRing":
        r = DelayedRing(float(self.scale))
        r.hist = self.hist.copy()
        r.idx = self.idx
        return r

    def fold(self, a, fmt: int) -> None:
        """Write amax into the window, advance, publish the next scale."""
        self.hist[self.idx] = np.float32(a)
        self.idx = (self.idx + 1) % HISTORY
        m = np.float32(np.max(self.hist))
        if m > 0 and np.isfinite(m):
            self.scale = _fmax_over(fmt, m)

    def step(self, x, fmt: int):
        """Quantize x with the current scale, then fold its amax.

        Returns (codes, amax, scale used by this call).
        """
        s = np.float32(self.scale)
        a = amax(x)
        q = quantize_with_scale(x, s, fmt)
        self.fold(a, fmt)
        return q, a, s

    def seed_step(self, x, fmt: int):
        """A seeded call: quantize x with its own current scale instead of
        the ring's, then fold its amax like any call (the reading taken of the
        ring's "seed" in ``astrai/extension/fp8.py @4dc5e923``, bullet on the
        _ScaleRing objects with update/seed: a ring's first step can measure
        its scale rather than start at the initial one).

        Returns (codes, amax, scale used by this call).
        """
        q, a, s = quantize_current(x, fmt)
        self.fold(a, fmt)
        return q, a, s
