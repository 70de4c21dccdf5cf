"""Python binding of the fp8lite C ABI (include/fp8lite.h).

Argument marshalling only: every step of quantization and of the GEMM runs in
the CUDA library ``libfp8lite.so`` built in this package directory. The
functions carry the C names and argument order; buffers may be given as
torch tensors (their ``data_ptr()`` is passed) or as integer device
addresses, and ``stream`` defaults to torch's current CUDA stream. A non-OK
status raises ``Fp8Error``. Importing fails loudly when the library has not
been built: there is no fallback path.
"""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8lite.so")

FP8_E4M3, FP8_E5M2 = 0, 1
FP8_NT, FP8_NN, FP8_TN = 0, 1, 2
FP8_OK = 0
FP8_ERR_INVALID_ARG = 1
FP8_ERR_ALIGNMENT = 2
FP8_ERR_UNSUPPORTED = 3
FP8_ERR_CUDA = 4
FP8_ERR_DEVICE_TIMEOUT = 5
FP8_RING_HISTORY = 16
FP8_RING_BYTES = 80
FP8_IN_BF16, FP8_IN_F16, FP8_IN_F32 = 0, 1, 2
FP8_QL_ROW, FP8_QL_COL, FP8_QL_BOTH = 0, 1, 2
FP8_QUANTIZE_SEED_RING = 1
FP8_QUANTIZE_DEFER_FOLD = 2


class Fp8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class fp8_ring(ctypes.Structure):
    """Host image of the device ring (80 bytes)."""
    _fields_ = [("hist", ctypes.c_float * FP8_RING_HISTORY), ("scale", ctypes.c_float),
                ("idx", ctypes.c_uint32), ("amax_bits", ctypes.c_uint32), ("ticket", ctypes.c_uint32)]


assert ctypes.sizeof(fp8_ring) == FP8_RING_BYTES

FP8_QUANTIZE_MAX_JOBS = 8
FP8_QUANTIZE_SMALL_MAX = 65536


class fp8_quantize_job(ctypes.Structure):
    """One job of fp8_quantize_many (pointers are device addresses)."""
    _fields_ = [("x", ctypes.c_void_p), ("n", ctypes.c_int64), ("fmt", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("ring", ctypes.c_void_p), ("out8", ctypes.c_void_p),
                ("amax_out", ctypes.c_void_p), ("scale_out", ctypes.c_void_p)]


assert ctypes.sizeof(fp8_quantize_job) == 56

FP8_MM_MAX_GROUP = 4


class fp8_mm_problem(ctypes.Structure):
    """One problem of fp8_mm_grouped (pointers are device addresses)."""
    _fields_ = [("a8", ctypes.c_void_p), ("b8", ctypes.c_void_p), ("sa", ctypes.c_void_p), ("sb", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("bias_scale", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("fmt_a", ctypes.c_int32),
                ("fmt_b", ctypes.c_int32), ("layout", ctypes.c_int32), ("bias_fmt", ctypes.c_int32)]


assert ctypes.sizeof(fp8_mm_problem) == 96


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python fp8_delayed_scaling_quantize_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    sig = {
        "fp8_status_string": (ctypes.c_char_p, [I]),
        "fp8_abi_version": (I, []),
        "fp8_ring_init": (I, [P, F, P]),
        "fp8_ring_get": (I, [P, P, P]),
        "fp8_ring_set": (I, [P, P, P]),
        "fp8_quantize": (I, [P, I64, I, P, P, P, P, P]),
        "fp8_quantize_ex": (I, [P, I, I64, I, P, ctypes.c_uint32, P, P, P, P]),
        "fp8_quantize_2d": (I, [P, I, I64, I64, I, P, ctypes.c_uint32, I, P, P, P, P, P]),
        "fp8_mm": (I, [P, I, P, I, P, P, I, I64, I64, I64, I64, I64, I64, I64, P, P, I, P, P]),
        "fp8_last_device_error": (I, []),
        "fp8_selftest_wait_timeout": (I, [ctypes.c_uint32, P]),
        "fp8_bias_grad": (I, [P, I64, I64, P, P]),
        "fp8_quantize_many": (I, [P, ctypes.c_int32, P]),
        "fp8_quantize_many_ex": (I, [P, ctypes.c_int32, ctypes.c_uint32, P]),
        "fp8_quantize_current_many": (I, [P, ctypes.c_int32, P]),
        "fp8_rings_fold": (I, [P, ctypes.c_int32, P, P]),
        "fp8_mm_ws": (I, [P, I, P, I, P, P, I, I64, I64, I64, I64, I64, I64, I64, P, P, I, P, P, ctypes.c_size_t,
                          ctypes.c_int32, P]),
        "fp8_mm_workspace_size": (ctypes.c_size_t, [I64, I64, I64, I64, I, ctypes.c_int32]),
        "fp8_mm_out8": (I, [P, I, P, I, P, P, I, I64, I64, I64, I64, I64, I64, I64, P, P, I, I, P, P, P, P, P]),
        "fp8_mm_splitk_static": (I, [P, I, P, I, P, P, I, I64, I64, I64, I64, I64, I64, I64, P, P, I, P,
                                     ctypes.c_int32, P]),
        "fp8_mm_grouped": (I, [P, ctypes.c_int32, P]),
    }
    for name, (res, args) in sig.items():
        try:
            fn = getattr(lib, name)
        except AttributeError:
            raise ImportError(f"{LIB_PATH} lacks {name}: it is stale; rebuild it with "
                              f"`python fp8_delayed_scaling_quantize_b200/build.py`") from None
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x or None
    return x.data_ptr() or None


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


def _check(status: int, where: str) -> int:
    if status != FP8_OK:
        raise Fp8Error(status, where)
    return status


def status_string(status: int) -> str:
    return lib.fp8_status_string(int(status)).decode()


def fp8_abi_version() -> int:
    return lib.fp8_abi_version()


def fp8_ring_init(ring, init_scale: float = 1.0, stream=None):
    return _check(lib.fp8_ring_init(_ptr(ring), float(init_scale), _stream(stream)), "fp8_ring_init")


def fp8_ring_get(ring, stream=None) -> fp8_ring:
    host = fp8_ring()
    _check(lib.fp8_ring_get(_ptr(ring), ctypes.byref(host), _stream(stream)), "fp8_ring_get")
    return host


def fp8_ring_set(ring, host: fp8_ring, stream=None):
    return _check(lib.fp8_ring_set(_ptr(ring), ctypes.byref(host), _stream(stream)), "fp8_ring_set")


def fp8_quantize(x, n, fmt, ring, out8, amax_out, scale_out, stream=None):
    return _check(lib.fp8_quantize(_ptr(x), int(n), int(fmt), _ptr(ring), _ptr(out8), _ptr(amax_out),
                                   _ptr(scale_out), _stream(stream)), "fp8_quantize")


def fp8_quantize_ex(x, dtype, n, fmt, ring, flags, out8, amax_out, scale_out, stream=None):
    return _check(lib.fp8_quantize_ex(_ptr(x), int(dtype), int(n), int(fmt), _ptr(ring), int(flags), _ptr(out8),
                                      _ptr(amax_out), _ptr(scale_out), _stream(stream)), "fp8_quantize_ex")


def fp8_quantize_2d(x, dtype, rows, cols, fmt, ring, flags, layout, out8, out8_t, amax_out, scale_out,
                    stream=None):
    return _check(lib.fp8_quantize_2d(_ptr(x), int(dtype), int(rows), int(cols), int(fmt), _ptr(ring), int(flags),
                                      int(layout), _ptr(out8), _ptr(out8_t), _ptr(amax_out), _ptr(scale_out),
                                      _stream(stream)), "fp8_quantize_2d")


def fp8_rings_fold(rings, count, fmts, stream=None):
    """Fold the accumulated amax of `count` consecutive rings; fmts: ints."""
    arr = (ctypes.c_int32 * max(len(fmts), 1))(*[int(f) for f in fmts])
    return _check(lib.fp8_rings_fold(_ptr(rings), int(count), ctypes.cast(arr, ctypes.c_void_p), _stream(stream)),
                  "fp8_rings_fold")


def _jobs(jobs):
    arr = (fp8_quantize_job * max(len(jobs), 1))()
    for i, job in enumerate(jobs):
        x, n, fmt, ring, out8, amax_out, scale_out = job[:7]
        dtype = job[7] if len(job) > 7 else FP8_IN_BF16
        arr[i] = fp8_quantize_job(_ptr(x), int(n), int(fmt), int(dtype), _ptr(ring), _ptr(out8), _ptr(amax_out),
                                  _ptr(scale_out))
    return arr


def fp8_quantize_current_many(jobs, stream=None):
    """jobs: sequence of (x, n, fmt, None, out8, amax_out, scale_out[, dtype]),
    each current-scaled; bf16/fp16 of at most FP8_QUANTIZE_SMALL_MAX elements."""
    return _check(lib.fp8_quantize_current_many(ctypes.cast(_jobs(jobs), ctypes.c_void_p), len(jobs),
                                                _stream(stream)), "fp8_quantize_current_many")


def fp8_quantize_many(jobs, stream=None, flags=0):
    """jobs: sequence of (x, n, fmt, ring, out8, amax_out, scale_out[, dtype])."""
    return _check(lib.fp8_quantize_many_ex(ctypes.cast(_jobs(jobs), ctypes.c_void_p), len(jobs), int(flags),
                                           _stream(stream)), "fp8_quantize_many")


def fp8_mm(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, stride_c, bias,
           bias_scale, bias_fmt, out, stream=None):
    return _check(lib.fp8_mm(_ptr(a8), int(fa), _ptr(b8), int(fb), _ptr(sa), _ptr(sb), int(layout),
                             int(M), int(N), int(K), int(batch), int(stride_a), int(stride_b),
                             int(stride_c), _ptr(bias), _ptr(bias_scale), int(bias_fmt), _ptr(out),
                             _stream(stream)), "fp8_mm")


def fp8_mm_ws(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, stride_c, bias,
              bias_scale, bias_fmt, out, workspace, split_k=0, workspace_bytes=None, stream=None):
    """fp8_mm that splits K `split_k` ways using `workspace` (a
    zero-initialised device buffer; its size defaults to the tensor's nbytes)."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _check(lib.fp8_mm_ws(_ptr(a8), int(fa), _ptr(b8), int(fb), _ptr(sa), _ptr(sb), int(layout),
                                int(M), int(N), int(K), int(batch), int(stride_a), int(stride_b),
                                int(stride_c), _ptr(bias), _ptr(bias_scale), int(bias_fmt), _ptr(out),
                                _ptr(workspace), int(workspace_bytes), int(split_k), _stream(stream)), "fp8_mm_ws")


def fp8_mm_out8(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, stride_c, bias,
                bias_scale, bias_fmt, out_fmt, out_ring, out8, out_amax, out_scale, stream=None):
    return _check(lib.fp8_mm_out8(_ptr(a8), int(fa), _ptr(b8), int(fb), _ptr(sa), _ptr(sb), int(layout),
                                  int(M), int(N), int(K), int(batch), int(stride_a), int(stride_b), int(stride_c),
                                  _ptr(bias), _ptr(bias_scale), int(bias_fmt), int(out_fmt), _ptr(out_ring),
                                  _ptr(out8), _ptr(out_amax), _ptr(out_scale), _stream(stream)), "fp8_mm_out8")


def fp8_mm_grouped(problems, stream=None):
    """problems: sequence of (a8, fa, b8, fb, sa, sb, layout, M, N, K, bias,
    bias_scale, bias_fmt, out), each as fp8_mm's arguments with batch 1."""
    arr = (fp8_mm_problem * max(len(problems), 1))()
    for i, (a8, fa, b8, fb, sa, sb, layout, M, N, K, bias, bias_scale, bias_fmt, out) in enumerate(problems):
        arr[i] = fp8_mm_problem(_ptr(a8), _ptr(b8), _ptr(sa), _ptr(sb), _ptr(bias), _ptr(bias_scale), _ptr(out),
                                int(M), int(N), int(K), int(fa), int(fb), int(layout), int(bias_fmt))
    return _check(lib.fp8_mm_grouped(ctypes.cast(arr, ctypes.c_void_p), len(problems), _stream(stream)),
                  "fp8_mm_grouped")


def fp8_mm_workspace_size(M, N, K, batch, layout, split_k):
    return int(lib.fp8_mm_workspace_size(int(M), int(N), int(K), int(batch), int(layout), int(split_k)))


def fp8_mm_splitk_static(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, stride_c, bias,
                         bias_scale, bias_fmt, out, split_k, stream=None):
    """Split-K fp8_mm on the library's own scratch (no workspace argument)."""
    return _check(lib.fp8_mm_splitk_static(_ptr(a8), int(fa), _ptr(b8), int(fb), _ptr(sa), _ptr(sb), int(layout),
                                           int(M), int(N), int(K), int(batch), int(stride_a), int(stride_b),
                                           int(stride_c), _ptr(bias), _ptr(bias_scale), int(bias_fmt), _ptr(out),
                                           int(split_k), _stream(stream)), "fp8_mm_splitk_static")


def fp8_last_device_error():
    return _check(lib.fp8_last_device_error(), "fp8_last_device_error")


def fp8_bias_grad(g, rows, cols, out, stream=None):
    return _check(lib.fp8_bias_grad(_ptr(g), int(rows), int(cols), _ptr(out), _stream(stream)), "fp8_bias_grad")


def fp8_selftest_wait_timeout(limit_us: int, stream=None):
    return _check(lib.fp8_selftest_wait_timeout(int(limit_us), _stream(stream)), "fp8_selftest_wait_timeout")


def raw_status(fn_name: str, *args) -> int:
    """Call a C entry point with pre-marshalled arguments and return its
    status without raising (used to test argument validation)."""
    return getattr(lib, fn_name)(*args)
