"""Seeded random sequences of quantize calls on one ring, against the
oracle bit for bit.

Each seed fixes a format and makes five calls, each drawing its input type
(bf16, fp16, fp32), size (empty, a few elements, up to 3.2 M, ragged), scale
of magnitudes (1e-4 .. 1e3, sometimes all zeros) and mode: current scaling,
a delayed call, a seeded call, or a deferred call followed by a fold. The
codes, amax and scale of every call and the whole ring after it equal the
oracle's (the oracle's ring makes the same calls).
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import E4M3, E5M2
import workloads as W

pytestmark = pytest.mark.gpu

DTYPES = {0: torch.bfloat16, 1: torch.float16, 2: torch.float32}


@pytest.fixture(scope="module")
def g():
    import gpu_util
    return gpu_util


def _oracle_codes(x, s, fmt):
    """The oracle's codes of every element; for 16-bit inputs the oracle runs
    once per distinct bit pattern present (quantizing is element by element)."""
    if x.dtype == torch.float32:
        return oracle.quantize_with_scale(x.numpy(), s, fmt)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    present = np.flatnonzero(np.bincount(bits, minlength=1 << 16))
    values = torch.from_numpy(present.astype(np.int32)).to(torch.int16).view(x.dtype).float().numpy()
    table = np.zeros(1 << 16, dtype=np.uint8)
    table[present] = oracle.quantize_with_scale(values, s, fmt)
    return table[bits]


def _input(rng, seed):
    dtype = int(rng.choice([0, 0, 1, 2]))
    kind = rng.choice(["empty", "few", "mid", "big"], p=[0.05, 0.2, 0.45, 0.3])
    n = {"empty": 0, "few": int(rng.integers(1, 5000)), "mid": int(rng.integers(5000, 300000)),
         "big": int(rng.integers(300000, 3_200_000 if dtype != 2 else 1_000_000))}[kind]
    sigma = float(10 ** rng.uniform(-4, 3))
    if rng.random() < 0.08:
        x = torch.zeros(n, dtype=DTYPES[dtype])
    elif dtype == 0:
        x = W.bf16_normal((n,), sigma, seed)
    else:
        x = W.f32_normal((n,), sigma, seed).to(DTYPES[dtype])
    return dtype, x


@pytest.mark.parametrize("seed", range(24))
def test_random_call_sequence(g, seed):
    import fp8_delayed_scaling_quantize_b200 as fp8
    rng = np.random.default_rng(41000 + seed)
    fmt = int(rng.integers(0, 2))
    ring = g.new_ring()
    ref = oracle.DelayedRing()
    for call in range(5):
        dtype, x = _input(rng, 42000 + 10 * seed + call)
        xf = x.float().numpy()
        mode = str(rng.choice(["current", "delayed", "delayed", "seed", "defer"]))
        what = f"call {call} {mode} dtype {dtype} n {x.numel()} fmt {fmt}"
        if mode == "current":
            q, amax, scale = g.quantize_ex(x.cuda(), dtype, fmt)
            a = oracle.amax(xf)
            s = oracle.current_scale(a, fmt)
        elif mode == "seed":
            # DelayedRing.seed_step's steps (current scale of x, then the fold),
            # with the codes taken per distinct input value below
            q, amax, scale = g.quantize_ex(x.cuda(), dtype, fmt, ring, fp8.FP8_QUANTIZE_SEED_RING)
            a = oracle.amax(xf)
            s = oracle.current_scale(a, fmt)
            ref.fold(a, fmt)
        else:
            s = np.float32(ref.scale)
            flags = fp8.FP8_QUANTIZE_DEFER_FOLD if mode == "defer" else 0
            q, amax, scale = g.quantize_ex(x.cuda(), dtype, fmt, ring, flags)
            a = oracle.amax(xf)
            if mode == "defer":
                assert g.ring_state(ring)[3] == int(np.float32(a).view(np.uint32)), what
                fp8.fp8_rings_fold(ring, 1, [fmt])
            ref.fold(a, fmt)
        n = x.numel()
        assert np.array_equal(g.codes(q)[:n], _oracle_codes(x, s, fmt)), what
        assert g.f32(scale)[0] == np.float32(s), what
        assert g.f32(amax)[0] == np.float32(a), what
        hist, rs, idx, acc, ticket = g.ring_state(ring)
        assert np.array_equal(hist, ref.hist) and rs == ref.scale and idx == ref.idx, what
        assert acc == 0 and ticket == 0, what
    assert fp8.fp8_last_device_error() == fp8.FP8_OK


@pytest.mark.parametrize("seed", range(16))
def test_random_grouped_jobs(g, seed):
    """fp8_quantize_many with 1 .. 8 drawn jobs (own ring, format, input type
    and size each), three calls in a row: every job equals the oracle's
    delayed call on its own ring, bit for bit."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    rng = np.random.default_rng(43000 + seed)
    count = int(rng.integers(1, 9))
    fmts = [int(v) for v in rng.integers(0, 2, count)]
    rings = [g.new_ring() for _ in range(count)]
    refs = [oracle.DelayedRing() for _ in range(count)]
    for call in range(3):
        drawn = [_input(rng, 44000 + 100 * seed + 10 * call + j) for j in range(count)]
        outs = [torch.empty(max(x.numel(), 1), dtype=torch.uint8, device="cuda") for _, x in drawn]
        amaxs = [torch.full((1,), -1.0, device="cuda") for _ in range(count)]
        scales = [torch.full((1,), -1.0, device="cuda") for _ in range(count)]
        xd = [x.cuda() if x.numel() else None for _, x in drawn]
        fp8.fp8_quantize_many([(xd[j], drawn[j][1].numel(), fmts[j], rings[j], outs[j] if xd[j] is not None else None,
                                amaxs[j], scales[j], drawn[j][0]) for j in range(count)])
        for j, (dtype, x) in enumerate(drawn):
            what = f"call {call} job {j} dtype {dtype} n {x.numel()} fmt {fmts[j]}"
            xf = x.float().numpy()
            s = np.float32(refs[j].scale)
            a = oracle.amax(xf)
            refs[j].fold(a, fmts[j])
            assert np.array_equal(g.codes(outs[j])[:x.numel()], _oracle_codes(x, s, fmts[j])), what
            assert g.f32(scales[j])[0] == s and g.f32(amaxs[j])[0] == np.float32(a), what
            hist, rs, idx, acc, ticket = g.ring_state(rings[j])
            assert np.array_equal(hist, refs[j].hist) and rs == refs[j].scale and idx == refs[j].idx, what
            assert acc == 0 and ticket == 0, what
    assert fp8.fp8_last_device_error() == fp8.FP8_OK


@pytest.mark.parametrize("seed", range(16))
def test_random_dual_quantize(g, seed):
    """fp8_quantize_2d on drawn shapes (multiples of 8), input types and
    layouts, delayed or current: the row-major codes are the oracle's and
    the transposed copy holds the same bytes."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    rng = np.random.default_rng(45000 + seed)
    fmt = int(rng.integers(0, 2))
    ring = g.new_ring() if rng.random() < 0.7 else None
    ref = oracle.DelayedRing()
    for call in range(3):
        rows, cols = (int(v) * 8 for v in rng.integers(1, 160, 2))
        dtype = int(rng.choice([0, 1, 2]))
        sigma = float(10 ** rng.uniform(-3, 2))
        seed_x = 46000 + 10 * seed + call
        x = (W.bf16_normal((rows, cols), sigma, seed_x) if dtype == 0
             else W.f32_normal((rows, cols), sigma, seed_x).to(DTYPES[dtype]))
        layout = int(rng.choice([fp8.FP8_QL_COL, fp8.FP8_QL_BOTH]))
        out = torch.full((rows * cols,), 0xAB, dtype=torch.uint8, device="cuda")
        out_t = torch.full((rows * cols,), 0xCD, dtype=torch.uint8, device="cuda")
        amax = torch.full((1,), -1.0, device="cuda")
        scale = torch.full((1,), -1.0, device="cuda")
        fp8.fp8_quantize_2d(x.cuda(), dtype, rows, cols, fmt, ring, 0, layout, out, out_t, amax, scale)
        xf = x.float().numpy().reshape(-1)
        a = oracle.amax(xf)
        if ring is None:
            s = oracle.current_scale(a, fmt)
        else:
            s = np.float32(ref.scale)
            ref.fold(a, fmt)
        want = _oracle_codes(x.reshape(-1), s, fmt)
        what = f"call {call} {rows}x{cols} dtype {dtype} layout {layout}"
        assert np.array_equal(g.codes(out_t).reshape(cols, rows), want.reshape(rows, cols).T), what
        if layout == fp8.FP8_QL_BOTH:
            assert np.array_equal(g.codes(out), want), what
        else:
            assert (g.codes(out) == 0xAB).all(), what
        assert g.f32(scale)[0] == np.float32(s) and g.f32(amax)[0] == np.float32(a), what
        if ring is not None:
            hist, rs, idx, acc, ticket = g.ring_state(ring)
            assert np.array_equal(hist, ref.hist) and rs == ref.scale and idx == ref.idx, what
            assert acc == 0 and ticket == 0, what
