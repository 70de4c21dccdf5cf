"""GPU parity of fp8_quantize (through the C ABI) against the CPU oracle.

Bar: bit-exact codes, amax, scale used and full ring state. NaN inputs are
excluded from the code comparison (the NaN reading is unpinned) but must map
to a NaN code.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import E4M3, E5M2
import workloads as W

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def g():
    import gpu_util
    return gpu_util


def _nan_code(c, fmt):
    return (c & 0x7F) == 0x7F if fmt == E4M3 else (c & 0x7F) > 0x7C


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_every_bf16_pattern_under_many_scales(g, fmt):
    import fp8_delayed_scaling_quantize_b200 as fp8
    xs = W.bf16_bit_patterns()
    xf = xs.float().numpy()
    finite = np.isfinite(xf)
    xd = xs.cuda()
    scales = [1.0, float(np.float32(448.0) / np.float32(3.0)), 2.0 ** -20, 1e-3, 3.0e38, 7.5,
              2.0 ** 40, float(np.nextafter(np.float32(1.0), np.float32(0.0)))]
    for s in scales:
        s32 = np.float32(s)
        ring = g.new_ring()
        host = fp8.fp8_ring()
        host.scale = float(s32)
        fp8.fp8_ring_set(ring, host)
        q, amax, scale = g.quantize(xd, fmt, ring)
        got = g.codes(q)
        want = oracle.quantize_with_scale(xf, s32, fmt)
        nan = np.isnan(xf)
        assert np.array_equal(got[~nan], want[~nan]), f"scale {s}"
        assert all(_nan_code(int(c), fmt) for c in got[nan])
        assert g.f32(scale)[0] == s32
        assert g.f32(amax)[0] == oracle.amax(xf)          # inf: the patterns hold +-inf
        hist, rs, idx, acc, ticket = g.ring_state(ring)
        assert hist[0] == np.inf and idx == 1 and acc == 0 and ticket == 0
        assert rs == s32                                   # non-finite window max keeps it
    # finite patterns only: the ring publishes fmt_max / amax
    ring = g.new_ring()
    xfin = xs[torch.from_numpy(finite)].contiguous()
    q, amax, scale = g.quantize(xfin.cuda(), fmt, ring)
    ref = oracle.DelayedRing()
    want, a, s = ref.step(xfin.float().numpy(), fmt)
    assert np.array_equal(g.codes(q), want)
    hist, rs, idx, _, _ = g.ring_state(ring)
    assert np.array_equal(hist, ref.hist) and rs == ref.scale and idx == ref.idx


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
@pytest.mark.parametrize("n", [0, 1, 7, 8, 15, 16, 17, 1000, 65535, 65536, 65537, 4096 * 37 + 5, (1 << 20) + 3])
def test_current_scaling_ragged_sizes(g, fmt, n):
    """Up to 65536 elements current scaling runs in one single-block launch,
    above it as an amax pass and a quantize pass: both against the oracle."""
    x = W.bf16_normal((n,), 0.7, 9000 + n)
    q, amax, scale = g.quantize(x.cuda(), fmt, None)
    want, a, s = oracle.quantize_current(x.float().numpy(), fmt)
    assert np.array_equal(g.codes(q), want)
    assert g.f32(amax)[0] == a
    assert g.f32(scale)[0] == s


def test_current_scaling_degenerate(g):
    z = torch.zeros(1000, dtype=torch.bfloat16)
    q, amax, scale = g.quantize(z.cuda(), E4M3, None)
    assert g.f32(amax)[0] == 0.0 and g.f32(scale)[0] == 1.0 and not g.codes(q).any()
    # smallest bf16 subnormal: 448 / 2^-133 overflows -> FLT_MAX
    t = torch.tensor([2.0 ** -133, 0.0], dtype=torch.bfloat16)
    q, amax, scale = g.quantize(t.cuda(), E4M3, None)
    want, a, s = oracle.quantize_current(t.float().numpy(), E4M3)
    assert g.f32(scale)[0] == s == np.finfo(np.float32).max
    assert np.array_equal(g.codes(q), want)


def test_current_many_small_jobs(g):
    """fp8_quantize_current_many: eight small tensors current-scaled in one
    launch (bf16 and fp16, both formats, empty, ragged, all zeros, and every
    bf16 bit pattern): each job's codes, amax and scale are the oracle's
    current scaling, and equal fp8_quantize_ex on that tensor alone."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    sizes = [65536, 0, 1, 7, 4097, 1000, 65535, 65536]
    dtypes = [0, 1, 0, 1, 0, 0, 1, 0]
    fmts = [E4M3, E5M2, E4M3, E4M3, E5M2, E4M3, E5M2, E5M2]
    xs = []
    for j, (n, dt) in enumerate(zip(sizes, dtypes)):
        x = W.f32_normal((n,), 10.0 ** (j - 3), 5200 + j).to(torch.bfloat16 if dt == 0 else torch.float16)
        xs.append(x)
    xs[5] = torch.zeros(1000, dtype=torch.bfloat16)
    xs[7] = W.bf16_bit_patterns()  # NaN and Inf included: amax = inf, so scale 1
    xd = [x.cuda() if x.numel() else None for x in xs]
    outs = [torch.empty(max(n, 1), dtype=torch.uint8, device="cuda") for n in sizes]
    amaxs = [torch.full((1,), -1.0, device="cuda") for _ in sizes]
    scales = [torch.full((1,), -1.0, device="cuda") for _ in sizes]
    fp8.fp8_quantize_current_many([(xd[j], sizes[j], fmts[j], None, outs[j] if sizes[j] else None, amaxs[j],
                                    scales[j], dtypes[j]) for j in range(len(sizes))])
    for j, x in enumerate(xs):
        n, what = sizes[j], f"job {j}"
        want, a, sc = oracle.quantize_current(x.float().numpy(), fmts[j])
        got = g.codes(outs[j])[:n]
        nan = _nan_code(want, fmts[j])
        assert np.array_equal(got[~nan], want[~nan]) and _nan_code(got[nan], fmts[j]).all(), what
        assert g.f32(amaxs[j])[0] == a and g.f32(scales[j])[0] == sc, what
        alone, a1, s1 = g.quantize_ex(x.cuda(), dtypes[j], fmts[j])
        assert np.array_equal(g.codes(alone)[:n], got), what
        assert g.f32(a1)[0] == g.f32(amaxs[j])[0] and g.f32(s1)[0] == g.f32(scales[j])[0], what
    # amax_out is optional
    fp8.fp8_quantize_current_many([(xd[0], sizes[0], fmts[0], None, outs[0], None, scales[0], dtypes[0])])
    assert g.f32(scales[0])[0] == oracle.quantize_current(xs[0].float().numpy(), fmts[0])[2]


def test_ring_hand_table_on_gpu(g):
    with open(os.path.join(GOLDEN, "ring_sequence.json")) as f:
        gold = json.load(f)
    ring = g.new_ring()
    for a, used, published, why in gold["steps"]:
        x = torch.tensor([a, -a / 2, a / 4, 0.0] * 1000, dtype=torch.bfloat16).cuda()
        _, amax, scale = g.quantize(x, gold["fmt"], ring)
        assert g.f32(amax)[0] == a, why
        assert g.f32(scale)[0] == np.float32(used), why
        assert g.ring_state(ring)[1] == np.float32(published), why
    assert g.ring_state(ring)[2] == gold["final_idx"]


def _oracle_codes_by_value(x_bf16, scale, fmt):
    """The oracle's codes for every element of a bf16 tensor. Quantizing is
    element by element, so the oracle runs once per distinct bf16 value
    present (at most 65536) and each element takes its value's code."""
    bits = x_bf16.reshape(-1).view(torch.int16).numpy().view(np.uint16)
    present = np.flatnonzero(np.bincount(bits, minlength=1 << 16))
    values = (present.astype(np.uint32) << 16).view(np.float32)
    table = np.zeros(1 << 16, dtype=np.uint8)
    table[present] = oracle.quantize_with_scale(values, scale, fmt)
    return table[bits]


def test_linear_stack_delayed_eight_steps(g):
    """Every x, W, g of the dim-1024 linear stack at 2048 tokens, 8 delayed
    steps with the per-step magnitude walk: every code, amax, scale and
    ring."""
    walk = W.stack_walk()
    rings = [[g.new_ring() for _ in range(3)] for _ in W.LINEARS]
    refs = [[oracle.DelayedRing() for _ in range(3)] for _ in W.LINEARS]
    for step in range(W.STACK_STEPS):
        tensors = W.stack_tensors(step, walk)
        for li, t in enumerate(tensors):
            for ri, (role, fmt) in enumerate((("x", E4M3), ("w", E4M3), ("g", E5M2))):
                xc = t[role].reshape(-1)
                q, amax, scale = g.quantize(xc.cuda(), fmt, rings[li][ri])
                xf = xc.float().numpy()
                s_used = np.float32(refs[li][ri].scale)
                a = oracle.amax(xf)
                refs[li][ri].fold(a, fmt)
                want = _oracle_codes_by_value(xc, s_used, fmt)
                assert np.array_equal(g.codes(q), want), (step, li, role)
                assert g.f32(amax)[0] == a and g.f32(scale)[0] == s_used
                hist, rs, ridx, acc, ticket = g.ring_state(rings[li][ri])
                assert np.array_equal(hist, refs[li][ri].hist) and rs == refs[li][ri].scale
                assert ridx == refs[li][ri].idx and acc == 0 and ticket == 0


def test_graph_replay_and_checkpoint(g):
    import fp8_delayed_scaling_quantize_b200 as fp8
    n = 3 * (1 << 18) + 11
    base = W.bf16_normal((n,), 1.0, 77).cuda()
    x = base.clone()
    ring = g.new_ring()
    out = torch.empty(n, dtype=torch.uint8, device="cuda")
    amax = torch.empty(1, device="cuda")
    scale = torch.empty(1, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            fp8.fp8_quantize(x, n, E4M3, ring, out, amax, scale, stream=stream)
    torch.cuda.synchronize()
    fp8.fp8_ring_init(ring, 1.0)
    ref = oracle.DelayedRing()
    factors = W.uniform(0.5, 2.0, 78, 20)
    saved = None
    for i in range(20):
        x.copy_((base.float() * float(factors[i]) * (i + 1)).to(torch.bfloat16))
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        want, a, s = ref.step(x.float().cpu().numpy(), E4M3)
        assert np.array_equal(g.codes(out), want), i
        assert g.f32(scale)[0] == s and g.f32(amax)[0] == a
        if i == 9:
            saved = fp8.fp8_ring_get(ring)
            saved_ref = ref.copy()
    # restore the step-9 checkpoint into a fresh ring and continue: identical
    ring2 = g.new_ring()
    fp8.fp8_ring_set(ring2, saved)
    x.copy_((base.float() * 3.0).to(torch.bfloat16))
    q2, _, s2 = g.quantize(x, E4M3, ring2)
    want, _, s = saved_ref.step(x.float().cpu().numpy(), E4M3)
    assert g.f32(s2)[0] == s and np.array_equal(g.codes(q2), want)
    del graph


def test_empty_input_folds_zero(g):
    ring = g.new_ring(2.5)
    q, amax, scale = g.quantize(torch.empty(0, dtype=torch.bfloat16, device="cuda"), E4M3, ring)
    hist, rs, idx, _, _ = g.ring_state(ring)
    assert g.f32(amax)[0] == 0.0 and g.f32(scale)[0] == np.float32(2.5)
    assert idx == 1 and rs == np.float32(2.5) and not hist.any()


def test_misaligned_input_is_rejected(g):
    import fp8_delayed_scaling_quantize_b200 as fp8
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(64, dtype=torch.uint8, device="cuda")
    amax = torch.empty(1, device="cuda")
    st = fp8.raw_status("fp8_quantize", x.data_ptr() + 2, 32, 0, None, out.data_ptr(),
                        amax.data_ptr(), amax.data_ptr(), None)
    assert st == fp8.FP8_ERR_ALIGNMENT


def test_quantize_many_matches_the_oracle_per_job(g):
    """One launch quantizing several tensors (mixed formats, ragged, empty)
    equals fp8_quantize on each, over repeated calls (rings evolve)."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    sizes = [(3 << 20) + 5, 1000, 0, (1 << 18) + 3, 4096 * 37]
    fmts = [E4M3, E5M2, E4M3, E5M2, E4M3]
    rings = [g.new_ring() for _ in sizes]
    refs = [oracle.DelayedRing() for _ in sizes]
    outs = [torch.empty(max(n, 1), dtype=torch.uint8, device="cuda") for n in sizes]
    amaxs = [torch.empty(1, device="cuda") for _ in sizes]
    scales = [torch.empty(1, device="cuda") for _ in sizes]
    for call in range(3):
        xs = [(W.bf16_normal((n,), 0.5, 8000 + 10 * call + j).float() * (j + 1) * (call + 1)).to(torch.bfloat16)
              for j, n in enumerate(sizes)]
        xd = [x.cuda() for x in xs]
        fp8.fp8_quantize_many([(xd[j] if sizes[j] else None, sizes[j], fmts[j], rings[j],
                                outs[j] if sizes[j] else None, amaxs[j], scales[j]) for j in range(len(sizes))])
        for j, n in enumerate(sizes):
            want, a, s = refs[j].step(xs[j].float().numpy(), fmts[j])
            assert np.array_equal(g.codes(outs[j])[:n], want), (call, j)
            assert g.f32(scales[j])[0] == s and g.f32(amaxs[j])[0] == a, (call, j)
            hist, rs, idx, acc, ticket = g.ring_state(rings[j])
            assert np.array_equal(hist, refs[j].hist) and rs == refs[j].scale and idx == refs[j].idx
            assert acc == 0 and ticket == 0


# ---------------------------------------------------- fp16 / fp32 inputs ---

@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_every_f16_pattern_under_many_scales(g, fmt):
    import fp8_delayed_scaling_quantize_b200 as fp8
    xs = W.f16_bit_patterns()
    xf = xs.float().numpy()
    nan = np.isnan(xf)
    xd = xs.cuda()
    for s in [1.0, 3.5, 2.0 ** -10, 1.0e4, 2.0 ** 20, 0.1]:
        s32 = np.float32(s)
        ring = g.new_ring()
        host = fp8.fp8_ring()
        host.scale = float(s32)
        fp8.fp8_ring_set(ring, host)
        q, amax, scale = g.quantize_ex(xd, fp8.FP8_IN_F16, fmt, ring)
        got = g.codes(q)
        want = oracle.quantize_with_scale(xf, s32, fmt)
        assert np.array_equal(got[~nan], want[~nan]), f"scale {s}"
        assert all(_nan_code(int(c), fmt) for c in got[nan])
        assert g.f32(scale)[0] == s32 and g.f32(amax)[0] == oracle.amax(xf)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_f32_inputs_over_the_whole_range(g, fmt):
    """fp32 values from subnormal to FLT_MAX with +-0 and +-inf mixed in:
    delayed (a given scale) and current scaling, on the finite-only copy too
    (so that the measured scale is not the amax = inf fallback)."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    n = (1 << 20) + 5
    x = W.f32_mixed(n, 6000 + fmt)
    xf = x.numpy()
    for s in [1.0, 2.0 ** -60, 2.0 ** 40, 7.0]:
        s32 = np.float32(s)
        ring = g.new_ring()
        host = fp8.fp8_ring()
        host.scale = float(s32)
        fp8.fp8_ring_set(ring, host)
        q, amax, scale = g.quantize_ex(x.cuda(), fp8.FP8_IN_F32, fmt, ring)
        assert np.array_equal(g.codes(q), oracle.quantize_with_scale(xf, s32, fmt)), f"scale {s}"
        assert g.f32(amax)[0] == oracle.amax(xf) == np.inf
    finite = x.clone()
    finite[~torch.isfinite(finite)] = 0.0
    for t in (x, finite):
        q, amax, scale = g.quantize_ex(t.cuda(), fp8.FP8_IN_F32, fmt, None)
        want, a, s = oracle.quantize_current(t.numpy(), fmt)
        assert np.array_equal(g.codes(q), want)
        assert g.f32(amax)[0] == a and g.f32(scale)[0] == s


@pytest.mark.parametrize("dtype", [1, 2])
@pytest.mark.parametrize("n", [1, 7, 9, 1000, 65536, 4096 * 37 + 5])
def test_f16_f32_ragged_sizes(g, dtype, n):
    import fp8_delayed_scaling_quantize_b200 as fp8
    x = W.bf16_normal((n,), 0.7, 9100 + n).float()
    x = x.to(torch.float16) if dtype == fp8.FP8_IN_F16 else x * 1.0001
    q, amax, scale = g.quantize_ex(x.cuda(), dtype, E4M3, None)
    want, a, s = oracle.quantize_current(x.float().numpy(), E4M3)
    assert np.array_equal(g.codes(q), want) and g.f32(amax)[0] == a and g.f32(scale)[0] == s
    ring = g.new_ring(2.0)
    ref = oracle.DelayedRing(2.0)
    for _ in range(2):
        q, amax, scale = g.quantize_ex(x.cuda(), dtype, E5M2, ring)
        want, a, s = ref.step(x.float().numpy(), E5M2)
        assert np.array_equal(g.codes(q), want) and g.f32(scale)[0] == s
    hist, rs, idx, _, _ = g.ring_state(ring)
    assert np.array_equal(hist, ref.hist) and rs == ref.scale and idx == ref.idx


def test_quantize_many_mixed_input_types(g):
    import fp8_delayed_scaling_quantize_b200 as fp8
    xs = [W.bf16_normal((70001,), 0.5, 9201), W.bf16_normal((4096 * 9,), 2.0, 9202).float().to(torch.float16),
          W.f32_mixed(1 << 18, 9203), W.bf16_normal((33,), 0.1, 9204).float()]
    dts = [fp8.FP8_IN_BF16, fp8.FP8_IN_F16, fp8.FP8_IN_F32, fp8.FP8_IN_F32]
    fmts = [E4M3, E5M2, E4M3, E5M2]
    rings = [g.new_ring(1.5) for _ in xs]
    refs = [oracle.DelayedRing(1.5) for _ in xs]
    outs = [torch.empty(x.numel(), dtype=torch.uint8, device="cuda") for x in xs]
    scs = [torch.empty(1, device="cuda") for _ in xs]
    xd = [x.cuda() for x in xs]
    for _ in range(2):
        fp8.fp8_quantize_many([(xd[j], xs[j].numel(), fmts[j], rings[j], outs[j], None, scs[j], dts[j])
                               for j in range(len(xs))])
        for j, x in enumerate(xs):
            want, a, s = refs[j].step(x.float().numpy(), fmts[j])
            assert np.array_equal(g.codes(outs[j]), want), j
            assert g.f32(scs[j])[0] == s
            hist, rs, idx, acc, ticket = g.ring_state(rings[j])
            assert np.array_equal(hist, refs[j].hist) and rs == refs[j].scale and acc == 0 and ticket == 0


@pytest.mark.parametrize("dtype", [0, 1, 2])
def test_seeded_first_call(g, dtype):
    """A fresh ring's seeded call quantizes with the input's own scale and
    folds its amax; the ordinary calls after it follow the oracle's ring."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    torch_dt = {0: torch.bfloat16, 1: torch.float16, 2: torch.float32}[dtype]
    ring = g.new_ring()
    ref = oracle.DelayedRing()
    for step in range(4):
        x = (W.bf16_normal((300001,), 0.03, 9300 + step).float() * (step + 1)).to(torch_dt)
        flags = fp8.FP8_QUANTIZE_SEED_RING if step == 0 else 0
        q, amax, scale = g.quantize_ex(x.cuda(), dtype, E4M3, ring, flags)
        xf = x.float().numpy()
        want, a, s = ref.seed_step(xf, E4M3) if step == 0 else ref.step(xf, E4M3)
        assert np.array_equal(g.codes(q), want), step
        assert g.f32(scale)[0] == s and g.f32(amax)[0] == a, step
        hist, rs, idx, acc, ticket = g.ring_state(ring)
        assert np.array_equal(hist, ref.hist) and rs == ref.scale and idx == ref.idx, step
        assert acc == 0 and ticket == 0


# ------------------------------------------------ transposed / dual codes ---

def _q2d(g, x, dtype, rows, cols, fmt, ring, flags, layout):
    import fp8_delayed_scaling_quantize_b200 as fp8
    n = rows * cols
    out = torch.full((max(n, 16),), 0xAB, dtype=torch.uint8, device="cuda")
    out_t = torch.full((max(n, 16),), 0xCD, dtype=torch.uint8, device="cuda")
    amax = torch.full((1,), -1.0, device="cuda")
    scale = torch.full((1,), -1.0, device="cuda")
    fp8.fp8_quantize_2d(x, dtype, rows, cols, fmt, ring, flags, layout, out, out_t, amax, scale)
    return out[:n], out_t[:n], amax, scale


@pytest.mark.parametrize("rows,cols", [(64, 64), (8, 8), (200, 136), (1024, 2056), (4096, 1024), (8, 4104)])
@pytest.mark.parametrize("dtype", [0, 1, 2])
def test_dual_quantize_byte_equality_and_oracle(g, rows, cols, dtype):
    """Both orientations from one pass hold the same bytes, the row-major copy
    is the oracle's codes, and the ring moves as for the flat quantize."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    torch_dt = {0: torch.bfloat16, 1: torch.float16, 2: torch.float32}[dtype]
    ring = g.new_ring()
    ref = oracle.DelayedRing()
    for step in range(3):
        x = (W.bf16_normal((rows, cols), 0.05, 9500 + rows + step).float() * (1 + step)).to(torch_dt)
        xd = x.cuda()
        out, out_t, amax, scale = _q2d(g, xd, dtype, rows, cols, E4M3, ring, 0, fp8.FP8_QL_BOTH)
        want, a, s = ref.step(x.float().numpy().reshape(-1), E4M3)
        got = g.codes(out)
        assert np.array_equal(got, want), step
        assert np.array_equal(g.codes(out_t).reshape(cols, rows), got.reshape(rows, cols).T), step
        assert g.f32(scale)[0] == s and g.f32(amax)[0] == a
        hist, rs, idx, acc, ticket = g.ring_state(ring)
        assert np.array_equal(hist, ref.hist) and rs == ref.scale and idx == ref.idx and acc == 0 and ticket == 0
    # the transposed copy alone: the same bytes, and the row-major buffer untouched
    ring2 = g.new_ring()
    ring2_ref = oracle.DelayedRing()
    out, out_t, _, scale = _q2d(g, xd, dtype, rows, cols, E4M3, ring2, 0, fp8.FP8_QL_COL)
    want, _, s = ring2_ref.step(x.float().numpy().reshape(-1), E4M3)
    assert np.array_equal(g.codes(out_t).reshape(cols, rows), want.reshape(rows, cols).T)
    assert (g.codes(out) == 0xAB).all() and g.f32(scale)[0] == s


@pytest.mark.parametrize("flags", [0, 1])
def test_dual_quantize_current_and_seeded(g, flags):
    import fp8_delayed_scaling_quantize_b200 as fp8
    rows, cols = 512, 776
    x = W.f32_mixed(rows * cols, 9600 + flags)
    x[~torch.isfinite(x)] = 0.0
    x = x.reshape(rows, cols)
    ring = g.new_ring() if flags else None
    out, out_t, amax, scale = _q2d(g, x.cuda(), fp8.FP8_IN_F32, rows, cols, E5M2, ring, flags, fp8.FP8_QL_BOTH)
    if flags:
        ref = oracle.DelayedRing()
        want, a, s = ref.seed_step(x.numpy().reshape(-1), E5M2)
        hist, rs, idx, _, _ = g.ring_state(ring)
        assert np.array_equal(hist, ref.hist) and rs == ref.scale and idx == ref.idx
    else:
        want, a, s = oracle.quantize_current(x.numpy().reshape(-1), E5M2)
    got = g.codes(out)
    assert np.array_equal(got, want)
    assert np.array_equal(g.codes(out_t).reshape(cols, rows), got.reshape(rows, cols).T)
    assert g.f32(amax)[0] == a and g.f32(scale)[0] == s


def test_dual_quantize_empty_and_row_layout(g):
    import fp8_delayed_scaling_quantize_b200 as fp8
    ring = g.new_ring(2.0)
    out, out_t, amax, scale = _q2d(g, None, 0, 0, 64, E4M3, ring, 0, fp8.FP8_QL_BOTH)
    hist, rs, idx, _, _ = g.ring_state(ring)
    assert idx == 1 and rs == np.float32(2.0) and g.f32(scale)[0] == np.float32(2.0)
    # FP8_QL_ROW is the flat quantize
    x = W.bf16_normal((96, 40), 1.0, 9700).cuda()
    out, _, _, _ = _q2d(g, x, 0, 96, 40, E4M3, None, 0, fp8.FP8_QL_ROW)
    want, _, _ = oracle.quantize_current(x.float().cpu().numpy().reshape(-1), E4M3)
    assert np.array_equal(g.codes(out), want)


# ------------------------------------------- data-parallel amax exchange ---

def _bits(a):
    return int(np.array([a], np.float32).view(np.int32)[0])


def test_deferred_fold_with_a_group_amax(g):
    """Deferred calls leave each ring's amax in its accumulator; with the
    group's amax written there (as the all-reduce would) one fp8_rings_fold
    folds all rings exactly as the oracle folds that amax. Without a remote
    contribution, deferred + fold equals a plain delayed call bit for bit."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    fmts = [E4M3, E4M3, E5M2]
    rings = torch.zeros(3, 20, dtype=torch.int32, device="cuda")
    for i in range(3):
        fp8.fp8_ring_init(rings[i], 1.0)
    twin = g.new_ring()  # plain delayed calls on ring 0's inputs
    refs = [oracle.DelayedRing() for _ in fmts]
    for step in range(4):
        xs = [(W.bf16_normal((50001 + 8 * i,), 0.02 * (i + 1), 9800 + 10 * step + i).float() * (step + 1))
              .to(torch.bfloat16) for i in range(3)]
        locals_ = []
        for i, x in enumerate(xs):
            q, amax, scale = g.quantize_ex(x.cuda(), 0, fmts[i], rings[i], fp8.FP8_QUANTIZE_DEFER_FOLD)
            xf = x.float().numpy()
            s_used = np.float32(refs[i].scale)
            assert np.array_equal(g.codes(q), oracle.quantize_with_scale(xf, s_used, fmts[i])), (step, i)
            assert g.f32(scale)[0] == s_used and g.f32(amax)[0] == oracle.amax(xf)
            locals_.append(np.float32(oracle.amax(xf)))
        # the all-reduce: another rank saw 3x the amax of role 1 (and less for role 2)
        group = [locals_[0], np.float32(locals_[1] * 3), locals_[2]]
        assert int(rings[1, 18]) == _bits(locals_[1])
        rings[1, 18] = _bits(group[1])
        rings[2, 18] = max(int(rings[2, 18]), _bits(locals_[2] / 2))
        fp8.fp8_rings_fold(rings, 3, fmts)
        for i in range(3):
            refs[i].fold(group[i], fmts[i])
            hist, rs, idx, acc, ticket = g.ring_state(rings[i])
            assert np.array_equal(hist, refs[i].hist) and rs == refs[i].scale and idx == refs[i].idx, (step, i)
            assert acc == 0 and ticket == 0
        # ring 0 had no remote contribution: it matches the plain delayed twin
        q_t, _, s_t = g.quantize(xs[0].cuda(), E4M3, twin)
        assert np.array_equal(g.ring_state(twin)[0], g.ring_state(rings[0])[0])
        assert g.ring_state(twin)[1] == g.ring_state(rings[0])[1]


def test_grouped_deferred_then_fold(g):
    import fp8_delayed_scaling_quantize_b200 as fp8
    sizes = [70001, 4096 * 5, 333]
    fmts = [E4M3, E5M2, E4M3]
    rings = torch.zeros(3, 20, dtype=torch.int32, device="cuda")
    for i in range(3):
        fp8.fp8_ring_init(rings[i], 1.0)
    refs = [oracle.DelayedRing() for _ in sizes]
    outs = [torch.empty(n, dtype=torch.uint8, device="cuda") for n in sizes]
    scs = [torch.empty(1, device="cuda") for _ in sizes]
    for step in range(3):
        xs = [W.bf16_normal((n,), 0.1 * (step + 1), 9900 + 10 * step + j) for j, n in enumerate(sizes)]
        xd = [x.cuda() for x in xs]
        fp8.fp8_quantize_many([(xd[j], sizes[j], fmts[j], rings[j], outs[j], None, scs[j]) for j in range(3)],
                              flags=fp8.FP8_QUANTIZE_DEFER_FOLD)
        fp8.fp8_rings_fold(rings, 3, fmts)
        for j in range(3):
            want, a, s = refs[j].step(xs[j].float().numpy(), fmts[j])
            assert np.array_equal(g.codes(outs[j]), want) and g.f32(scs[j])[0] == s
            hist, rs, idx, acc, ticket = g.ring_state(rings[j])
            assert np.array_equal(hist, refs[j].hist) and rs == refs[j].scale and acc == 0 and ticket == 0


def test_exchange_helper_on_one_rank(g):
    """The torch.distributed helper end to end on a one-rank NCCL group (the
    all-reduce is then the identity): deferred calls, exchange, fold."""
    import socket
    import torch.distributed as dist
    import fp8_delayed_scaling_quantize_b200 as fp8
    from fp8_delayed_scaling_quantize_b200.dist import allreduce_amax_and_fold
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        rings = torch.zeros(2, 20, dtype=torch.int32, device="cuda")
        for i in range(2):
            fp8.fp8_ring_init(rings[i], 1.0)
        refs = [oracle.DelayedRing(), oracle.DelayedRing()]
        x = W.bf16_normal((12345,), 0.3, 9950)
        for i, fmt in enumerate((E4M3, E5M2)):
            g.quantize_ex(x.cuda(), 0, fmt, rings[i], fp8.FP8_QUANTIZE_DEFER_FOLD)
            refs[i].fold(oracle.amax(x.float().numpy()), fmt)
        allreduce_amax_and_fold(rings, [E4M3, E5M2])
        torch.cuda.synchronize()
        for i in range(2):
            hist, rs, idx, acc, _ = g.ring_state(rings[i])
            assert np.array_equal(hist, refs[i].hist) and rs == refs[i].scale and acc == 0
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_more_than_2_to_31_elements(g, fmt):
    """A tensor past 2^31 elements (4 GB of bf16, with a ragged tail): every
    bf16 bit pattern repeated, quantized with a delayed scale. Every code
    equals the oracle's code of the same pattern, the amax is +inf (the
    infinite patterns; NaN is ignored) and the ring keeps its scale, as the
    oracle's ring does."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    n = (1 << 31) + 19
    pats = W.bf16_bit_patterns()
    x = pats.cuda().repeat(n // 65536 + 1)[:n].contiguous()
    s = np.float32(2.0 ** -4)
    ring = g.new_ring()
    host = fp8.fp8_ring()
    host.scale = float(s)
    fp8.fp8_ring_set(ring, host)
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    amax = torch.empty(1, device="cuda")
    sc = torch.empty(1, device="cuda")
    fp8.fp8_quantize(x, n, fmt, ring, q, amax, sc)
    want = oracle.quantize_with_scale(pats.float().numpy(), s, fmt)
    # element i holds pattern i mod 65536: every code is checked on the device
    # against the oracle's code of its pattern (any NaN code where the
    # oracle's is NaN), a block of whole repetitions at a time
    want_dev = torch.from_numpy(want).cuda()
    nan_col = torch.from_numpy(_nan_code(want, fmt)).cuda()
    codes = np.arange(256, dtype=np.uint8)
    nan_codes = torch.from_numpy(codes[_nan_code(codes, fmt)]).cuda()
    reps = n // 65536
    rows = q[:reps * 65536].view(reps, 65536)
    for r0 in range(0, reps, 2048):
        blk = rows[r0:r0 + 2048]
        ok = (blk == want_dev) | (nan_col & torch.isin(blk, nan_codes))
        assert bool(ok.all()), f"rows {r0}..{r0 + blk.shape[0]}"
    tail = q[reps * 65536:]
    ok = (tail == want_dev[:tail.numel()]) | (nan_col[:tail.numel()] & torch.isin(tail, nan_codes))
    assert tail.numel() == 19 and bool(ok.all())
    assert g.f32(sc)[0] == s and g.f32(amax)[0] == np.inf
    r = oracle.DelayedRing(float(s))
    r.fold(np.float32(np.inf), fmt)
    hist, rs, idx_, acc, ticket = g.ring_state(ring)
    assert np.array_equal(hist, r.hist) and rs == r.scale and idx_ == r.idx and acc == 0 and ticket == 0
    del x, q
    torch.cuda.empty_cache()
