"""Pins for the oracle's amax, scales and delayed ring (CPU only).

Pinned against: brute-force maxima, closed-form scales at powers of two,
the property that a tensor's largest element lands on the top code, the
hand-computed ring table in tests/golden/ring_sequence.json, and the
"no scale-ratio leak" regression of the AstrAI commit log
(astrai/extension/fp8.py @f4c44ebf: two delayed steps with a changing amax).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import E4M3, E5M2
from workloads import bf16_normal

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FLT_MAX = float(np.finfo(np.float32).max)


def _f32(t):
    return t.float().numpy()


def test_amax_brute_force():
    x = _f32(bf16_normal((3, 1001), 3.0, 1))
    want = 0.0
    for v in x.reshape(-1).tolist():
        want = max(want, abs(v))
    assert float(oracle.amax(x)) == want
    assert float(oracle.amax(np.zeros(0, np.float32))) == 0.0
    # the largest magnitude may be negative
    y = np.array([1.0, -7.5, 3.0], np.float32)
    assert float(oracle.amax(y)) == 7.5


def test_amax_is_taken_before_quantization():
    """The amax bug: measuring the quantized max (about 448) collapses the scale."""
    x = np.array([0.001, -0.002, 0.0005], np.float32)
    ring = oracle.DelayedRing()
    ring.step(x, E4M3)
    assert float(oracle.amax(x)) == np.float32(0.002)
    assert ring.hist[0] == np.float32(0.002)
    assert float(ring.scale) > 1000.0


@pytest.mark.parametrize("k", [-20, -3, 0, 1, 5, 14])
def test_current_scale_powers_of_two(k):
    a = 2.0 ** k
    assert float(oracle.current_scale(a, E4M3)) == 448.0 * 2.0 ** -k
    assert float(oracle.current_scale(a, E5M2)) == 57344.0 * 2.0 ** -k


def test_current_scale_degenerate():
    assert float(oracle.current_scale(0.0, E4M3)) == 1.0
    assert float(oracle.current_scale(math.inf, E4M3)) == 1.0
    # 448 / 2^-133 overflows fp32: clamped to the largest finite value
    assert float(oracle.current_scale(2.0 ** -133, E4M3)) == FLT_MAX


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_current_scaling_puts_the_max_on_the_top_code(fmt, seed):
    x = _f32(bf16_normal((4096,), 0.37 * seed, seed))
    q, a, s = oracle.quantize_current(x, fmt)
    i = int(np.argmax(np.abs(x)))
    top = 0x7E if fmt == E4M3 else 0x7B
    assert int(q[i]) & 0x7F == top
    # and no code exceeds the top code
    assert int(np.max(q & 0x7F)) <= top
    # the dequantized tensor is close to the input (relative step of the format)
    deq = oracle.decode_table(fmt)[q] / float(s)
    rel = 2.0 ** -4 if fmt == E4M3 else 2.0 ** -3
    big = np.abs(x) > float(a) * 2 ** -6
    assert np.all(np.abs(deq[big] - x[big]) <= rel * np.abs(x[big]))


def test_quantize_product_is_rounded_to_fp32_once():
    """x*s is rounded to fp32 first, then to FP8: two roundings, in that order.

    x = 1.0078125 (bf16 0x3F81) and s = fp32 0x3F06F21C: the exact product is
    0.53125 + 1.3e-8, just above the E4M3 tie between 0.5 (0x30) and 0.5625
    (0x31), but its fp32 rounding is the tie itself, which goes to the even
    code 0x30. Rounding the exact product straight to FP8 would give 0x31.
    """
    from fractions import Fraction
    x = np.float32(1.0078125)
    s = np.array([0x3F06F21C], np.uint32).view(np.float32)[0]
    exact = Fraction(float(x)) * Fraction(float(s))
    assert exact > Fraction(17, 32)
    assert np.float32(float(exact)) == np.float32(0.53125)
    assert int(oracle.quantize_with_scale(np.array([x]), s, E4M3)[0]) == 0x30


def test_ring_matches_hand_computed_table():
    with open(os.path.join(GOLDEN, "ring_sequence.json")) as f:
        g = json.load(f)
    ring = oracle.DelayedRing()
    for a, used, published, why in g["steps"]:
        # a tensor whose amax is exactly a (values bf16-representable)
        x = np.array([a, -a / 2, a / 4, 0.0], np.float32)
        _, got_a, got_used = ring.step(x, g["fmt"])
        assert float(got_a) == a
        assert float(got_used) == used, why
        assert float(ring.scale) == np.float32(published), why
    assert ring.idx == g["final_idx"]

    r5 = oracle.DelayedRing()
    r5.step(np.array([g["e5m2_step"]["amax"]], np.float32), E5M2)
    assert float(r5.scale) == g["e5m2_step"]["published"]

    ro = oracle.DelayedRing()
    tiny = np.float32(2.0 ** g["overflow_step"]["amax_log2"])
    assert tiny > 0
    ro.step(np.array([tiny], np.float32), E4M3)
    assert float(ro.scale) == g["overflow_step"]["published"]


def test_ring_zero_amax_keeps_scale_and_window_wraps():
    ring = oracle.DelayedRing(init_scale=3.0)
    ring.step(np.zeros(8, np.float32), E4M3)
    assert float(ring.scale) == 3.0 and ring.idx == 1
    for _ in range(16):
        ring.step(np.ones(2, np.float32), E4M3)
    assert ring.idx == 1 and np.all(ring.hist == 1.0) and float(ring.scale) == 448.0


def test_no_scale_ratio_leak_between_delayed_steps():
    """Two delayed steps with a changing amax: each step's GEMM must match
    the real product when dequantized with the scales the quantize USED, and
    would be off by the scale ratio with the freshly published ones."""
    rx, rw = oracle.DelayedRing(), oracle.DelayedRing()
    x1 = _f32(bf16_normal((16, 64), 1.0, 31))
    w1 = _f32(bf16_normal((8, 64), 1.0, 32))
    # step 2: 1.5x the magnitude (mild saturation under step 1's scale)
    x2 = _f32((torch.from_numpy(x1) * 1.5).to(torch.bfloat16))
    w2 = _f32((torch.from_numpy(w1) * 1.5).to(torch.bfloat16))
    for x, w in ((x1, w1), (x2, w2)):
        qx, _, sx = rx.step(x, E4M3)
        qw, _, sw = rw.step(w, E4M3)
        assert float(sx) != float(rx.scale) and float(sw) != float(rw.scale)
        true = x.astype(np.float64) @ w.astype(np.float64).T
        y, _ = oracle.mm(qx, E4M3, qw, E4M3, sx, sw, oracle.NT, 16, 8, 64)
        err = np.linalg.norm(y[0] - true) / np.linalg.norm(true)
        assert err < 0.1, err
        ratio = float(sx) * float(sw) / (float(rx.scale) * float(rw.scale))
        y_bad, _ = oracle.mm(qx, E4M3, qw, E4M3, rx.scale, rw.scale, oracle.NT, 16, 8, 64)
        got = np.linalg.norm(y_bad[0]) / np.linalg.norm(true)
        assert abs(got / ratio - 1.0) < 0.1 and abs(ratio - 1.0) > 0.5


def test_seeded_step_closed_forms():
    """Fresh ring, x = [2, -1, 0.5, 0]: the seeded call scales by 448 / 2 = 224
    (every product exactly representable in E4M3, so decoding the codes and
    dividing by 224 gives x back exactly), writes 2 into hist[0], advances idx
    to 1 and publishes 224; the next ordinary call uses 224. Seeding a ring
    that already has history folds into hist[idx], not hist[0]."""
    x = np.array([2.0, -1.0, 0.5, 0.0], np.float32)
    r = oracle.DelayedRing()
    q, a, s = r.seed_step(x, E4M3)
    assert a == np.float32(2.0) and s == np.float32(224.0)
    assert np.array_equal(oracle.decode_table(E4M3)[q] / np.float32(224.0), x)
    assert r.hist[0] == np.float32(2.0) and not r.hist[1:].any() and r.idx == 1
    assert r.scale == np.float32(224.0)
    q2, a2, s2 = r.step(np.array([4.0], np.float32), E4M3)
    assert s2 == np.float32(224.0) and r.scale == np.float32(112.0)  # window max 4 -> 448 / 4
    # a ring with history: the seed folds at idx, and the window keeps the old maximum
    r3 = oracle.DelayedRing()
    r3.fold(np.float32(8.0), E4M3)
    _, _, s3 = r3.seed_step(x, E4M3)
    assert s3 == np.float32(224.0) and r3.hist[1] == np.float32(2.0) and r3.idx == 2
    assert r3.scale == np.float32(56.0)  # 448 / max(8, 2)
    # zero input: current scale 1, and the zero amax keeps the ring's scale
    r4 = oracle.DelayedRing(3.0)
    q4, a4, s4 = r4.seed_step(np.zeros(5, np.float32), E5M2)
    assert s4 == np.float32(1.0) and a4 == 0 and r4.scale == np.float32(3.0) and not q4.any()
