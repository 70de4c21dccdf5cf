"""The C-ABI library loads, exports every declared entry point, and rejects
bad arguments on the host before any launch (CPU only: no compute call)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fp8():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "fp8lite_build", os.path.join(ROOT, "fp8_delayed_scaling_quantize_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    build.build()
    import fp8_delayed_scaling_quantize_b200 as m
    return m


def _declared():
    with open(os.path.join(ROOT, "include", "fp8lite.h")) as f:
        text = f.read()
    return re.findall(r"FP8LITE_API\s+[\w\s\*]+?\b(fp8_\w+)\s*\(", text)


def test_every_declared_symbol_is_exported(fp8):
    names = _declared()
    assert len(names) >= 8
    lib = ctypes.CDLL(fp8.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_abi_version_and_status_strings(fp8):
    assert fp8.fp8_abi_version() == 4
    for code, name in [(0, "FP8_OK"), (1, "FP8_ERR_INVALID_ARG"), (2, "FP8_ERR_ALIGNMENT"),
                       (3, "FP8_ERR_UNSUPPORTED"), (4, "FP8_ERR_CUDA"), (5, "FP8_ERR_DEVICE_TIMEOUT")]:
        assert fp8.status_string(code) == name


# Fake device addresses: the host validation must reject before touching them.
A = 0x7F0000000000
S = 0x7F0000100000


def q(fp8, x=A, n=64, fmt=0, ring=None, out=A + 4096, amax=S, scale=S + 4):
    return fp8.raw_status("fp8_quantize", x, n, fmt, ring, out, amax, scale, None)


def test_quantize_validation(fp8):
    assert q(fp8, fmt=2) == fp8.FP8_ERR_INVALID_ARG
    assert q(fp8, fmt=-1) == fp8.FP8_ERR_INVALID_ARG
    assert q(fp8, n=-1) == fp8.FP8_ERR_INVALID_ARG
    assert q(fp8, n=1 << 40) == fp8.FP8_ERR_INVALID_ARG
    assert q(fp8, scale=None) == fp8.FP8_ERR_INVALID_ARG
    assert q(fp8, x=None) == fp8.FP8_ERR_INVALID_ARG
    assert q(fp8, out=None) == fp8.FP8_ERR_INVALID_ARG
    assert q(fp8, amax=None) == fp8.FP8_ERR_INVALID_ARG  # current scaling needs it
    assert q(fp8, x=A + 2) == fp8.FP8_ERR_ALIGNMENT
    assert q(fp8, out=A + 4096 + 8) == fp8.FP8_ERR_ALIGNMENT
    assert q(fp8, ring=S + 2) == fp8.FP8_ERR_ALIGNMENT
    assert q(fp8, scale=S + 1) == fp8.FP8_ERR_ALIGNMENT


def mm(fp8, a8=A, fa=0, b8=A + 65536, fb=0, sa=S, sb=S + 4, layout=0, M=128, N=128, K=128,
       batch=1, stride_a=0, stride_b=0, stride_c=0, bias=None, bias_scale=None, bias_fmt=0,
       out=A + 262144):
    return fp8.raw_status("fp8_mm", a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a,
                          stride_b, stride_c, bias, bias_scale, bias_fmt, out, None)


def test_mm_validation(fp8):
    E, AL, U = fp8.FP8_ERR_INVALID_ARG, fp8.FP8_ERR_ALIGNMENT, fp8.FP8_ERR_UNSUPPORTED
    assert mm(fp8, fa=3) == E
    assert mm(fp8, layout=3) == E
    assert mm(fp8, a8=None) == E
    assert mm(fp8, sa=None) == E
    assert mm(fp8, out=None) == E
    assert mm(fp8, M=0) == E and mm(fp8, N=0) == E and mm(fp8, K=0) == E
    assert mm(fp8, batch=0) == E
    assert mm(fp8, stride_a=-16, batch=2, stride_c=128 * 128) == E
    assert mm(fp8, bias_scale=S + 8) == E            # a scale without a bias
    assert mm(fp8, batch=2, stride_c=100) == E       # overlapping outputs
    assert mm(fp8, M=1 << 31) == U
    # TMA row pitch: K (NT), N for B (NN/TN), M for A (TN) multiples of 16
    assert mm(fp8, K=100) == AL
    assert mm(fp8, layout=1, N=100) == AL
    assert mm(fp8, layout=2, M=100) == AL
    assert mm(fp8, a8=A + 8) == AL
    assert mm(fp8, batch=2, stride_a=8, stride_c=1 << 20) == AL
    assert mm(fp8, out=A + 262144 + 2) == AL
    # free dimensions: M and N in NT need no alignment (checked up to launch:
    # every check above must fail before any CUDA call on this CPU-only host)


def test_ring_validation(fp8):
    assert fp8.raw_status("fp8_ring_init", None, ctypes.c_float(1.0), None) == fp8.FP8_ERR_INVALID_ARG
    assert fp8.raw_status("fp8_ring_init", S, ctypes.c_float(0.0), None) == fp8.FP8_ERR_INVALID_ARG
    assert fp8.raw_status("fp8_ring_init", S, ctypes.c_float(float("inf")), None) == fp8.FP8_ERR_INVALID_ARG
    assert fp8.raw_status("fp8_ring_init", S + 2, ctypes.c_float(1.0), None) == fp8.FP8_ERR_ALIGNMENT
    host = fp8.fp8_ring()
    host.idx = 16
    host.scale = 1.0
    assert fp8.raw_status("fp8_ring_set", S, ctypes.byref(host), None) == fp8.FP8_ERR_INVALID_ARG
    assert fp8.raw_status("fp8_ring_get", None, ctypes.byref(host), None) == fp8.FP8_ERR_INVALID_ARG


def test_quantize_many_validation(fp8):
    def status(jobs, count=None):
        arr = (fp8.fp8_quantize_job * max(len(jobs), 1))(*[fp8.fp8_quantize_job(*j) for j in jobs])
        return fp8.raw_status("fp8_quantize_many", ctypes.cast(arr, ctypes.c_void_p),
                              len(jobs) if count is None else count, None)
    good = (A, 64, 0, 0, S, A + 4096, None, S + 64)   # x, n, fmt, dtype, ring, out8, amax_out, scale_out
    assert status([good], count=0) == fp8.FP8_ERR_INVALID_ARG
    assert status([good] * 9) == fp8.FP8_ERR_INVALID_ARG
    assert status([good, good]) == fp8.FP8_ERR_INVALID_ARG                       # one ring twice
    assert status([(A, 64, 0, 0, None, A + 4096, None, S + 64)]) == fp8.FP8_ERR_INVALID_ARG  # no ring
    assert status([(A, 64, 5, 0, S, A + 4096, None, S + 64)]) == fp8.FP8_ERR_INVALID_ARG     # bad fmt
    assert status([(A, 64, 0, 3, S, A + 4096, None, S + 64)]) == fp8.FP8_ERR_INVALID_ARG     # bad dtype
    assert status([(A + 2, 64, 0, 0, S, A + 4096, None, S + 64)]) == fp8.FP8_ERR_ALIGNMENT
    assert fp8.raw_status("fp8_quantize_many", None, 1, None) == fp8.FP8_ERR_INVALID_ARG


def test_quantize_current_many_validation(fp8):
    def status(jobs, count=None):
        arr = (fp8.fp8_quantize_job * max(len(jobs), 1))(*[fp8.fp8_quantize_job(*j) for j in jobs])
        return fp8.raw_status("fp8_quantize_current_many", ctypes.cast(arr, ctypes.c_void_p),
                              len(jobs) if count is None else count, None)
    good = (A, 64, 0, 0, None, A + 4096, None, S + 64)   # x, n, fmt, dtype, ring, out8, amax_out, scale_out
    assert status([good], count=0) == fp8.FP8_ERR_INVALID_ARG
    assert status([good] * 9) == fp8.FP8_ERR_INVALID_ARG
    assert status([(A, 64, 0, 0, S, A + 4096, None, S + 64)]) == fp8.FP8_ERR_INVALID_ARG      # a ring given
    assert status([(A, 64, 0, 0, None, A + 4096, None, None)]) == fp8.FP8_ERR_INVALID_ARG    # no scale_out
    assert status([(None, 64, 0, 0, None, A + 4096, None, S + 64)]) == fp8.FP8_ERR_INVALID_ARG  # no x
    assert status([(A, 64, 2, 0, None, A + 4096, None, S + 64)]) == fp8.FP8_ERR_INVALID_ARG  # bad fmt
    assert status([(A, 64, 0, 2, None, A + 4096, None, S + 64)]) == fp8.FP8_ERR_UNSUPPORTED  # fp32 input
    assert status([(A, fp8.FP8_QUANTIZE_SMALL_MAX + 8, 0, 0, None, A + (1 << 20), None, S + 64)]) == \
        fp8.FP8_ERR_UNSUPPORTED
    assert status([(A + 8, 64, 0, 0, None, A + 4096, None, S + 64)]) == fp8.FP8_ERR_ALIGNMENT
    assert status([(A, 64, 0, 0, None, A + 4096, S + 2, S + 64)]) == fp8.FP8_ERR_ALIGNMENT


def test_mm_workspace_size_and_alignment(fp8):
    # no split requested or chosen: no workspace
    assert fp8.fp8_mm_workspace_size(2048, 1024, 4096, 1, fp8.FP8_NT, 0) == 0
    assert fp8.fp8_mm_workspace_size(2048, 1024, 4096, 1, fp8.FP8_NT, 1) == 0
    # two splits: the counters plus at least two fp32 partials of the whole output
    assert fp8.fp8_mm_workspace_size(2048, 1024, 4096, 1, fp8.FP8_NT, 2) >= 4096 + 2 * 2048 * 1024 * 4
    # one row: swapped operands, partial tiles of 16 rows (M padded to 16, not 128)
    assert fp8.fp8_mm_workspace_size(1, 4096, 4096, 1, fp8.FP8_NT, 4) == 4096 + 4 * 16 * 4096 * 4
    # too many tile halves for the counters, too few k-blocks, bad arguments
    assert fp8.fp8_mm_workspace_size(8192, 8192, 8192, 1, fp8.FP8_NT, 2) == 0
    assert fp8.fp8_mm_workspace_size(2048, 1024, 256, 1, fp8.FP8_NT, 4) == 0
    assert fp8.fp8_mm_workspace_size(0, 8, 8, 1, fp8.FP8_NT, 2) == 0
    assert fp8.fp8_mm_workspace_size(8, 8, 8, 1, 7, 2) == 0
    assert fp8.fp8_mm_workspace_size(8, 8, 1024, 1, fp8.FP8_NT, 5) == 0
    st = fp8.raw_status("fp8_mm_ws", A, 0, A, 0, S, S, 0, 16, 16, 16, 1, 256, 256, 256, None, None, 0, A,
                        A + 8, 1 << 20, 2, None)
    assert st == fp8.FP8_ERR_ALIGNMENT
    st = fp8.raw_status("fp8_mm_ws", A, 0, A, 0, S, S, 9, 16, 16, 16, 1, 256, 256, 256, None, None, 0, A,
                        A, 1 << 20, 2, None)
    assert st == fp8.FP8_ERR_INVALID_ARG
    for split_k in (-1, 5):
        st = fp8.raw_status("fp8_mm_ws", A, 0, A, 0, S, S, 0, 16, 16, 16, 1, 256, 256, 256, None, None, 0, A,
                            A, 1 << 20, split_k, None)
        assert st == fp8.FP8_ERR_INVALID_ARG


def test_quantize_ex_validation(fp8):
    def st(x=A, dtype=0, n=64, fmt=0, ring=S, flags=0, out8=A + 4096, amax=S + 128, scale=S + 64):
        return fp8.raw_status("fp8_quantize_ex", x, dtype, n, fmt, ring, flags, out8, amax, scale, None)
    assert st(dtype=3) == fp8.FP8_ERR_INVALID_ARG
    assert st(dtype=-1) == fp8.FP8_ERR_INVALID_ARG
    assert st(flags=4) == fp8.FP8_ERR_INVALID_ARG                        # unknown flag
    assert st(flags=3) == fp8.FP8_ERR_INVALID_ARG                        # seed and deferred fold together
    assert st(ring=None, flags=fp8.FP8_QUANTIZE_DEFER_FOLD, amax=S + 128) == fp8.FP8_ERR_INVALID_ARG
    assert st(ring=None, flags=fp8.FP8_QUANTIZE_SEED_RING) == fp8.FP8_ERR_INVALID_ARG  # seed needs a ring
    assert st(flags=fp8.FP8_QUANTIZE_SEED_RING, amax=None) == fp8.FP8_ERR_INVALID_ARG  # seed needs amax_out
    assert st(ring=None, amax=None) == fp8.FP8_ERR_INVALID_ARG           # current scaling needs amax_out
    assert st(x=A + 4, dtype=2) == fp8.FP8_ERR_ALIGNMENT                 # fp32 input still 16-byte aligned
    assert st(fmt=7) == fp8.FP8_ERR_INVALID_ARG


def test_quantize_2d_validation(fp8):
    def st(rows=64, cols=64, layout=2, ring=S, flags=0, out8=A + 4096, out8_t=A + 8192, dtype=0, amax=S + 128):
        return fp8.raw_status("fp8_quantize_2d", A, dtype, rows, cols, 0, ring, flags, layout, out8, out8_t, amax,
                              S + 64, None)
    assert st(layout=3) == fp8.FP8_ERR_INVALID_ARG
    assert st(rows=-8) == fp8.FP8_ERR_INVALID_ARG
    assert st(rows=60) == fp8.FP8_ERR_ALIGNMENT            # the transposed copy needs multiples of 8
    assert st(cols=12) == fp8.FP8_ERR_ALIGNMENT
    assert st(out8_t=None) == fp8.FP8_ERR_INVALID_ARG
    assert st(layout=2, out8=None) == fp8.FP8_ERR_INVALID_ARG
    assert st(layout=1, out8=None, out8_t=A + 8200) == fp8.FP8_ERR_ALIGNMENT
    assert st(ring=None, flags=1) == fp8.FP8_ERR_INVALID_ARG
    assert st(dtype=5) == fp8.FP8_ERR_INVALID_ARG


def test_rings_fold_and_grouped_flags_validation(fmt_ok=(0, 1)):
    import fp8_delayed_scaling_quantize_b200 as fp8
    arr = (ctypes.c_int32 * 3)(0, 1, 0)
    assert fp8.raw_status("fp8_rings_fold", None, 3, ctypes.cast(arr, ctypes.c_void_p), None) == fp8.FP8_ERR_INVALID_ARG
    assert fp8.raw_status("fp8_rings_fold", S, 0, ctypes.cast(arr, ctypes.c_void_p), None) == fp8.FP8_ERR_INVALID_ARG
    assert fp8.raw_status("fp8_rings_fold", S, 65, ctypes.cast(arr, ctypes.c_void_p), None) == fp8.FP8_ERR_INVALID_ARG
    assert fp8.raw_status("fp8_rings_fold", S, 3, None, None) == fp8.FP8_ERR_INVALID_ARG
    bad = (ctypes.c_int32 * 3)(0, 7, 0)
    assert fp8.raw_status("fp8_rings_fold", S, 3, ctypes.cast(bad, ctypes.c_void_p), None) == fp8.FP8_ERR_INVALID_ARG
    assert fp8.raw_status("fp8_rings_fold", S + 2, 3, ctypes.cast(arr, ctypes.c_void_p), None) == fp8.FP8_ERR_ALIGNMENT
    jobs = (fp8.fp8_quantize_job * 1)(fp8.fp8_quantize_job(A, 64, 0, 0, S, A + 4096, None, S + 64))
    assert fp8.raw_status("fp8_quantize_many_ex", ctypes.cast(jobs, ctypes.c_void_p), 1, 1, None) == \
        fp8.FP8_ERR_INVALID_ARG  # the seed is not offered for grouped calls


def test_mm_out8_validation(fp8):
    def st(out_fmt=0, ring=S, out8=A + 8192, scale=S + 64, amax=None):
        return fp8.raw_status("fp8_mm_out8", A, 0, A, 0, S, S, 0, 16, 16, 16, 1, 256, 256, 256, None, None, 0,
                              out_fmt, ring, out8, amax, scale, None)
    assert st(out_fmt=3) == fp8.FP8_ERR_INVALID_ARG
    assert st(ring=None) == fp8.FP8_ERR_INVALID_ARG
    assert st(scale=None) == fp8.FP8_ERR_INVALID_ARG
    assert st(out8=None) == fp8.FP8_ERR_INVALID_ARG
    assert st(ring=S + 2) == fp8.FP8_ERR_ALIGNMENT


def test_mm_grouped_validation(fp8):
    def prob(**kw):
        d = dict(a8=A, b8=A, sa=S, sb=S, bias=None, bias_scale=None, out=A + 262144, M=128, N=128, K=128,
                 fmt_a=0, fmt_b=0, layout=0, bias_fmt=0)
        d.update(kw)
        return fp8.fp8_mm_problem(**d)

    def st(probs, count=None):
        arr = (fp8.fp8_mm_problem * max(len(probs), 1))(*probs)
        return fp8.raw_status("fp8_mm_grouped", ctypes.cast(arr, ctypes.c_void_p),
                              len(probs) if count is None else count, None)
    E, AL, U = fp8.FP8_ERR_INVALID_ARG, fp8.FP8_ERR_ALIGNMENT, fp8.FP8_ERR_UNSUPPORTED
    assert fp8.raw_status("fp8_mm_grouped", None, 1, None) == E
    assert st([prob()], count=0) == E
    assert st([prob()] * (fp8.FP8_MM_MAX_GROUP + 1)) == E
    assert st([prob(), prob(fmt_a=3)]) == E           # the second problem decides
    assert st([prob(layout=3)]) == E
    assert st([prob(out=None)]) == E and st([prob(sb=None)]) == E
    assert st([prob(), prob(M=0)]) == E and st([prob(K=0)]) == E
    assert st([prob(bias_scale=S + 8)]) == E           # a scale without a bias
    assert st([prob(bias=A, bias_scale=S + 8, bias_fmt=7)]) == E
    assert st([prob(N=1 << 31)]) == U
    assert st([prob(K=100)]) == AL                     # TMA row pitches, as fp8_mm
    assert st([prob(layout=1, N=100)]) == AL
    assert st([prob(layout=2, M=100)]) == AL
    assert st([prob(), prob(b8=A + 8)]) == AL
    assert st([prob(out=A + 2)]) == AL
