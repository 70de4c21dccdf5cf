"""Benchmark of the FP8 linear-layer hot path on B200.

One step = one pass of the whole path over the dim-1024 transformer linear
stack at 2048 tokens (B4 x T512): for each of the 4 linears (QKV 1024->3072,
out 1024->1024, MLP 1024->4096, 4096->1024) delayed-scaling quantize of x
and W to E4M3 and of the gradient g to E5M2 (ring finalized in-kernel),
then the forward NT GEMM y = x W^T, the dX NN GEMM g W and the dW TN GEMM
g^T x, all through the C ABI: 8 GEMM launches (a forward per linear, and one
grouped launch per linear for its dX and dW; --no-group-bwd: 12 single GEMMs)
and 8 quantize launches (one grouped launch for every W and the first x, then
each later x and every g; --no-grouped: 12 single-tensor quantize launches).

value  = GEMM FLOPs of the step (154.6 GFLOP) / device step time, TFLOP/s,
         the step replayed as one CUDA graph (16 kernel nodes), inputs
         resident in HBM, rotating through 3 input sets (276 MB > 126 MB L2).
e2e    = the same metric through the public API with HOST buffers: pinned
         host -> device copies of x, W, g and device -> host copies of y,
         dX, dW inside the timed region, eager calls; the copies of
         consecutive steps overlap (double buffers, one copy stream each way).
roofline / roofline_quantize = the GEMM kernel and the quantize kernel,
         each timed per launch with CUDA events on the launching stream.
cpu_baseline = the CPU oracle (numpy, fp64 GEMM) on one full step.

--impl reference times the oracle on the host cores instead (a bounded
sample of the same step per bench step).
"""

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "FP8 GEMM TFLOP/s & quantize GB/s on 1 B200, % of roofline"
WORKLOAD = "linear stack dim1024 tokens2048 (B4xT512): QKV/out/MLP-up/MLP-down, fwd NT + dX NN + dW TN, delayed rings H=16"
N_SETS = 3
E4M3, E5M2 = 0, 1
NT, NN, TN = 0, 1, 2


KERNEL_SOURCES = {
    "gemm": ("gemm.cu", "sm100.cuh", "common.cuh"),
    "quantize": ("quantize.cu", "common.cuh"),
}


def source_hash(kind):
    """sha256 over the CUDA sources a kernel family is built from."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "fp8_delayed_scaling_quantize_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(kind):
    """DRAM bytes per launch from the committed ncu capture summary, or None
    when the kernel's sources changed since the capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)[kind]
    except Exception:
        return None
    return t["dram_bytes_per_launch"] if t.get("source_sha256") == source_hash(kind) else None


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------ distributed ---

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def weak_scaling_value(flops_per_step, steps, world, t_ms_max):
    """Whole-job TFLOP/s: every rank runs `steps` steps of its own replica;
    the job takes the slowest rank's time."""
    return flops_per_step * steps * world / (t_ms_max * 1e-3) / 1e12


def max_over_ranks(v, world):
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- clocks ---

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
             0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
             0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index, period=0.01):
        self.period = period
        self.samples = []
        self.reasons = 0
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        names = [n for bit, n in self.NAMES.items() if self.reasons & bit]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------- the stack ---

class Stack:
    """Device buffers and the C-ABI calls of one step of the linear stack."""

    def __init__(self, fp8, n_sets=N_SETS, dev="cuda", tokens=W.TOKENS):
        """tokens: a multiple of the workload's 2048; above it, each set's x
        and g are the workload's draws repeated along the token dimension (the
        values do not change the timing)."""
        self.fp8 = fp8
        self.dev = dev
        self.tokens = tokens
        rep = tokens // W.TOKENS
        assert rep * W.TOKENS == tokens
        self.sets = []
        for s in range(n_sets):
            ts = W.stack_tensors(s)
            self.sets.append([{k: (v.to(dev).repeat(rep, 1) if k != "w" and rep > 1 else v.to(dev))
                               for k, v in t.items()} for t in ts])
        T = tokens
        self.lin = []
        # all 12 rings in one [12, 20] tensor, so the data-parallel exchange
        # all-reduces their amax words in one message and folds them in one launch
        self.rings = torch.empty(3 * len(W.LINEARS), 20, dtype=torch.int32, device=dev)
        self.ring_fmts = [E4M3, E4M3, E5M2] * len(W.LINEARS)
        self.dp_amax = False
        for li, (name, d_in, d_out) in enumerate(W.LINEARS):
            L = {"name": name, "d_in": d_in, "d_out": d_out}
            L["q"] = {r: torch.empty(n, dtype=torch.uint8, device=dev)
                      for r, n in (("x", T * d_in), ("w", d_out * d_in), ("g", T * d_out))}
            L["ring"] = {r: self.rings[3 * li + k] for k, r in enumerate(("x", "w", "g"))}
            for r in L["ring"].values():
                fp8.fp8_ring_init(r, 1.0)
            L["scale"] = {r: torch.empty(1, device=dev) for r in ("x", "w", "g")}
            L["amax"] = {r: torch.empty(1, device=dev) for r in ("x", "w", "g")}
            L["y"] = torch.empty(T * d_out, dtype=torch.bfloat16, device=dev)
            L["dx"] = torch.empty(T * d_in, dtype=torch.bfloat16, device=dev)
            L["dw"] = torch.empty(d_out * d_in, dtype=torch.bfloat16, device=dev)
            self.lin.append(L)
        self.flops = sum(3 * 2 * T * di * do for _, di, do in W.LINEARS)
        self.q_elems = sum(T * di + do * di + T * do for _, di, do in W.LINEARS)
        self.split_k = 0
        self.ws = [None, None]
        self.group_bwd = True

    def use_group_bwd(self):
        """dX and dW of a linear in one fp8_mm_grouped launch (not with split K)."""
        return self.group_bwd and self.split_k <= 1

    def bwd_pair(self, li):
        """dX and dW of linear li as the two problems of one grouped launch."""
        _, dx, dw = self.gemm_calls(li)
        return [c[:10] + c[14:18] for c in (dx, dw)]

    def use_split(self, split_k):
        """Run every GEMM of the step that can take it with split_k K-splits,
        one zero-filled workspace per stream."""
        self.split_k = split_k
        if split_k > 1:
            need = max(self.fp8.fp8_mm_workspace_size(*c[7:11], c[6], split_k) for li in range(len(self.lin))
                       for c in self.gemm_calls(li))
            self.ws = [torch.zeros(max(need, 4096), dtype=torch.uint8, device=self.dev) for _ in range(2)]

    def quantize(self, call, stream):
        if self.dp_amax:
            x, n, fmt, ring, out8, amax, scale = call
            self.fp8.fp8_quantize_ex(x, 0, n, fmt, ring, self.fp8.FP8_QUANTIZE_DEFER_FOLD, out8, amax, scale,
                                     stream=stream)
        else:
            self.fp8.fp8_quantize(*call, stream=stream)

    def exchange(self, stream):
        """The data-parallel amax exchange at the end of a step: all-reduce the
        12 rings' amax words over the ranks (none with one rank), one fold."""
        import torch.distributed as dist
        from fp8_delayed_scaling_quantize_b200.dist import allreduce_amax
        with torch.cuda.stream(stream):
            if dist.is_initialized() and dist.get_world_size() > 1:
                allreduce_amax(self.rings)
            self.fp8.fp8_rings_fold(self.rings, self.rings.shape[0], self.ring_fmts, stream=stream)

    def mm(self, call, stream, ws_index=0):
        c = call
        if self.split_k > 1 and self.fp8.fp8_mm_workspace_size(*c[7:11], c[6], self.split_k) > 0:
            self.fp8.fp8_mm_ws(*call, self.ws[ws_index], self.split_k, stream=stream)
        else:
            self.fp8.fp8_mm(*call, stream=stream)

    def quant_calls(self, s, li):
        L, t = self.lin[li], self.sets[s][li]
        return [(t[r], t[r].numel(), fmt, L["ring"][r], L["q"][r], L["amax"][r], L["scale"][r])
                for r, fmt in (("x", E4M3), ("w", E4M3), ("g", E5M2))]

    def gemm_calls(self, li):
        L = self.lin[li]
        T, di, do = self.tokens, L["d_in"], L["d_out"]
        q, sc = L["q"], L["scale"]
        return [
            # forward y = x W^T: NT, M=T, N=d_out, K=d_in
            (q["x"], E4M3, q["w"], E4M3, sc["x"], sc["w"], NT, T, do, di, 1, 0, 0, 0, None, None, 0, L["y"]),
            # dX = g W: NN, M=T, N=d_in, K=d_out
            (q["g"], E5M2, q["w"], E4M3, sc["g"], sc["w"], NN, T, di, do, 1, 0, 0, 0, None, None, 0, L["dx"]),
            # dW = g^T x: TN, M=d_out, N=d_in, K=T
            (q["g"], E5M2, q["x"], E4M3, sc["g"], sc["x"], TN, do, di, T, 1, 0, 0, 0, None, None, 0, L["dw"]),
        ]

    def gemm_flops(self, li):
        L = self.lin[li]
        return 2 * self.tokens * L["d_in"] * L["d_out"]

    def grouped_call(self, s):
        """The step-start quantize of every linear's W and of the first x,
        as the jobs of one fp8_quantize_many launch."""
        return [self.quant_calls(s, li)[1] for li in range(len(self.lin))] + [self.quant_calls(s, 0)[0]]

    def step(self, s, stream, side=None, grouped=True):
        """Issue one training step of the stack on input set s: the forward
        of every linear in order (quantize x and W, y = x W^T), then the
        backward in reverse order (quantize g, dX = g W, dW = g^T x).

        grouped: the weights are all known when the step starts, so every W
        and the first x are quantized by one grouped launch; the x of later
        linears and every g still wait for the layer before them.
        The backward's dX and dW (both only need g8) run as one grouped GEMM
        launch; without it (split K, or --no-group-bwd) and with a `side`
        stream, dW runs on that stream beside dX. A `side` stream also takes
        W's quantize beside x's (ungrouped). The streams fork and join around
        each pair, so the dependencies between linears are those of a
        sequential model."""
        fp8 = self.fp8
        n = len(self.lin)
        if grouped:
            fp8.fp8_quantize_many(self.grouped_call(s), stream=stream,
                                  flags=fp8.FP8_QUANTIZE_DEFER_FOLD if self.dp_amax else 0)
        for li in range(n):
            qx, qw, _ = self.quant_calls(s, li)
            fwd, _, _ = self.gemm_calls(li)
            if grouped:
                if li > 0:
                    self.quantize(qx, stream)
            elif side is not None:
                side.wait_stream(stream)
                self.quantize(qw, side)
                self.quantize(qx, stream)
                stream.wait_stream(side)
            else:
                self.quantize(qx, stream)
                self.quantize(qw, stream)
            self.mm(fwd, stream)
        for li in reversed(range(n)):
            _, _, qg = self.quant_calls(s, li)
            _, dx, dw = self.gemm_calls(li)
            self.quantize(qg, stream)
            if self.use_group_bwd():
                fp8.fp8_mm_grouped(self.bwd_pair(li), stream=stream)
            elif side is not None:
                side.wait_stream(stream)
                self.mm(dw, side, 1)
                self.mm(dx, stream, 0)
                stream.wait_stream(side)
            else:
                self.mm(dx, stream)
                self.mm(dw, stream)
        if self.dp_amax:
            self.exchange(stream)

    def launches_per_step(self, grouped=True):
        n = len(self.lin)
        gemms = n + (n if self.use_group_bwd() else 2 * n)
        return gemms + (1 + (n - 1) + n if grouped else 3 * n) + (1 if self.dp_amax else 0)


def hold_stream(stream, us=2000):
    """Park the stream in a device-side sleep while the host enqueues the
    next launches, so that event pairs around each launch time the kernel,
    not the host's submission gaps."""
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(us * 1965))


def gemm_algorithmic_bytes(layout, M, N, K):
    """Compulsory HBM bytes of one GEMM launch: operands once, bf16 out once."""
    return M * K + N * K + 2 * M * N


def breakdown(fp8, stack, stream, reps, rotate):
    """Per-launch device time of each of the step's kernels, back to back.

    rotate=False repeats each call on the step's own buffers (L2-resident);
    rotate=True gives call i copies number i mod k of every input and output,
    k sized so that the copies exceed twice the L2, so each launch reads its
    inputs from HBM as it does inside the step."""
    dev = stack.dev
    q_ms = g_ms = 0.0
    q_elems = g_flops = g_bytes = 0
    n_g = n_q = 0
    per_shape, per_tensor = {}, {}
    names = ("x", "w", "g")
    for li in range(len(stack.lin)):
        L = stack.lin[li]
        calls = [("quantize", c, names[i]) for i, c in enumerate(stack.quant_calls(0, li))]
        if stack.use_group_bwd():
            calls += [("gemm", stack.gemm_calls(li)[0], None), ("pair", stack.bwd_pair(li), None)]
        else:
            calls += [("gemm", c, None) for c in stack.gemm_calls(li)]
        for kind, c, role in calls:
            if kind == "quantize":
                x, n, fmt, ring, q, am, sc = c
                k = _slots(3 * n) if rotate else 1
                X = [x] + [x.clone() for _ in range(k - 1)]
                Q = [q] + [torch.empty_like(q) for _ in range(k - 1)]
                call = lambda i: fp8.fp8_quantize(X[i % k], n, fmt, ring, Q[i % k], am, sc, stream=stream)
            elif kind == "pair":
                dx, dw = c
                g8, w8, x8 = dx[0], dx[2], dw[2]
                nbytes = g8.numel() + w8.numel() + x8.numel() + 2 * (dx[13].numel() + dw[13].numel())
                k = _slots(nbytes) if rotate else 1
                G = [g8] + [g8.clone() for _ in range(k - 1)]
                Wc = [w8] + [w8.clone() for _ in range(k - 1)]
                Xc = [x8] + [x8.clone() for _ in range(k - 1)]
                DX = [dx[13]] + [torch.empty_like(dx[13]) for _ in range(k - 1)]
                DW = [dw[13]] + [torch.empty_like(dw[13]) for _ in range(k - 1)]
                call = lambda i: fp8.fp8_mm_grouped(
                    [(G[i % k],) + dx[1:2] + (Wc[i % k],) + dx[3:13] + (DX[i % k],),
                     (G[i % k],) + dw[1:2] + (Xc[i % k],) + dw[3:13] + (DW[i % k],)], stream=stream)
            else:
                M, N, K = c[7:10]
                k = _slots(gemm_algorithmic_bytes(c[6], M, N, K)) if rotate else 1
                A = [c[0]] + [c[0].clone() for _ in range(k - 1)]
                B = [c[2]] + [c[2].clone() for _ in range(k - 1)]
                C = [c[17]] + [torch.empty_like(c[17]) for _ in range(k - 1)]
                call = lambda i: stack.mm((A[i % k],) + c[1:2] + (B[i % k],) + c[3:17] + (C[i % k],), stream)
            ms = _time_us(stream, call, reps) * 1e-3
            if kind == "quantize":
                q_ms += ms
                q_elems += c[1]
                n_q += 1
                per_tensor[f"{L['name']}.{role} {c[1]}"] = (ms, c[1])
            elif kind == "pair":
                g_ms += ms
                f = sum(2 * M * N * K for (M, N, K) in (q[7:10] for q in c))
                g_flops += f
                g_bytes += sum(gemm_algorithmic_bytes(q[6], *q[7:10]) for q in c)
                n_g += 1
                per_shape[" + ".join(f"{'NT NN TN'.split()[q[6]]} {q[7]}x{q[8]}x{q[9]}" for q in c)] = (ms, f)
            else:
                M, N, K = c[7:10]
                g_ms += ms
                g_flops += 2 * M * N * K
                g_bytes += gemm_algorithmic_bytes(c[6], M, N, K)
                n_g += 1
                per_shape[f"{'NT NN TN'.split()[c[6]]} {M}x{N}x{K}"] = (ms, 2 * M * N * K)
    torch.cuda.synchronize()
    return {"q_ms": q_ms, "q_elems": q_elems, "n_q": n_q, "g_ms": g_ms, "g_flops": g_flops, "g_bytes": g_bytes,
            "n_g": n_g, "per_shape": per_shape, "per_tensor": per_tensor}


# ------------------------------------------------------------ our arm -------

def run_ours(args, world, rank, local):
    import fp8_delayed_scaling_quantize_b200 as fp8
    hbm, bf16_burst, bf16_sust, peak_src = _peaks()
    fp8_burst = 2.0 * bf16_burst      # dense FP8 = 2x dense bf16 (nominal 4.5 / 2.25 PF/s)
    stream = torch.cuda.Stream()
    side = None if args.one_stream else torch.cuda.Stream()
    stack = Stack(fp8)
    stack.use_split(args.split_k)
    stack.dp_amax = args.dp_amax
    stack.group_bwd = not args.no_group_bwd
    grouped = not args.no_grouped
    torch.cuda.synchronize()

    # warm-up (eager) also sets kernel attributes before any capture
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            stack.step(i % N_SETS, stream, side, grouped)
    torch.cuda.synchronize()

    graphs = []
    if not args.no_graph:
        for s in range(N_SETS):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                stack.step(s, stream, side, grouped)
            graphs.append(g)
        torch.cuda.synchronize()
        for i in range(max(args.warmup, 3)):
            with torch.cuda.stream(stream):
                graphs[i % N_SETS].replay()
        torch.cuda.synchronize()

    # ---- timed region -------------------------------------------------
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(args.steps):
                if graphs:
                    graphs[i % N_SETS].replay()
                else:
                    stack.step(i % N_SETS, stream, side, grouped)
            e1.record(stream)
        e1.synchronize()
    torch.cuda.synchronize()
    used_graphs = bool(graphs)
    graphs.clear()  # released before anything else: they may hold NCCL calls (--dp-amax)
    barrier(world)
    t_ms = max_over_ranks(e0.elapsed_time(e1), world)
    ms_step = t_ms / args.steps
    value = weak_scaling_value(stack.flops, args.steps, world, t_ms)

    # ---- per-kernel breakdown -----------------------------------------
    # Each of the step's 12 quantizes and its GEMM launches (a forward per
    # linear, and a grouped dX + dW launch per linear, or the two apart) is
    # repeated back to back between one event pair (the stream held while the
    # host enqueues), so the average is the kernel's steady-state cost on the
    # stream, as inside the graph. The roofline figures rotate every call over
    # copies of its inputs and outputs that together exceed twice the L2 (HBM
    # traffic, as in the step, where a whole step's bytes pass between two uses
    # of one tensor); the same calls on one L2-resident set are reported apart.
    hot = breakdown(fp8, stack, stream, args.breakdown_reps, rotate=False)
    cold = breakdown(fp8, stack, stream, args.breakdown_reps, rotate=True)
    q_ms, q_elems, n_q = cold["q_ms"], cold["q_elems"], cold["n_q"]
    g_ms, g_flops, g_bytes, n_g = cold["g_ms"], cold["g_flops"], cold["g_bytes"], cold["n_g"]
    # the grouped step-start launch (all W + the first x) against its
    # tensors quantized one launch each
    jobs = stack.grouped_call(0)
    reps = args.breakdown_reps
    hold_stream(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fp8.fp8_quantize_many(jobs, stream=stream)
    e1.record(stream)
    e1.synchronize()
    many_ms = e0.elapsed_time(e1) / reps
    many_elems = sum(j[1] for j in jobs)
    hold_stream(stream)
    e0.record(stream)
    for _ in range(reps):
        for j in jobs:
            fp8.fp8_quantize(*j, stream=stream)
    e1.record(stream)
    e1.synchronize()
    single_ms = e0.elapsed_time(e1) / reps
    grouped_detail = {"jobs": len(jobs), "elems": many_elems, "us": round(1e3 * many_ms, 2),
                      "gbs": round(3.0 * many_elems / (many_ms * 1e-3) / 1e9, 1),
                      "frac": round(3.0 * many_elems / (many_ms * 1e-3) / 1e9 / hbm, 4),
                      "same_tensors_one_launch_each_us": round(1e3 * single_ms, 2),
                      "l2": "one input set (14.7 M elements, 29 MB bf16): L2-resident"}
    gemm_tf = g_flops / (g_ms * 1e-3) / 1e12
    quant_gbs = 3.0 * q_elems / (q_ms * 1e-3) / 1e9
    gemm_detail = {k: {"us": round(1e3 * ms, 2), "tflops": round(f / (ms * 1e-3) / 1e12, 1),
                       "us_l2_hot": round(1e3 * hot["per_shape"][k][0], 2)}
                   for k, (ms, f) in cold["per_shape"].items()}
    quant_detail = {k: {"us": round(1e3 * ms, 2), "gbs": round(3.0 * n / (ms * 1e-3) / 1e9, 1),
                        "us_l2_hot": round(1e3 * hot["per_tensor"][k][0], 2)}
                    for k, (ms, n) in cold["per_tensor"].items()}
    l2_hot = {"gemm_avg_launch_us": round(1e3 * hot["g_ms"] / hot["n_g"], 2),
              "gemm_tflops": round(hot["g_flops"] / (hot["g_ms"] * 1e-3) / 1e12, 1),
              "quantize_avg_launch_us": round(1e3 * hot["q_ms"] / hot["n_q"], 2),
              "quantize_gbs": round(3.0 * hot["q_elems"] / (hot["q_ms"] * 1e-3) / 1e9, 1),
              "method": "the same calls repeated on one input set (every tensor fits in the 126 MB L2)"}
    configs = None
    if not args.no_configs:
        with ClockSampler(local) as cfg_clocks:
            configs = run_configs(fp8, stream, hbm, fp8_burst)
        configs["clocks"] = cfg_clocks.summary()

    # ---- e2e: host buffers through the public API ------------------------
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(fp8, stack, stream, args.e2e_steps, world, side, grouped)
        e2e["value"] = round(e2e["value"], 3)

    context = {}
    if not args.no_compare:
        context = compare_bf16(stack, ms_step, 200)
        context["at_16384_tokens"] = compare_at_tokens(fp8, 8 * W.TOKENS, 50)
    gpu_launches = stack.launches_per_step(grouped) * args.steps
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8 e4m3/e5m2 operands, fp32 accumulate, bf16 out",
        "data": "synthetic (seeded bf16 normals of the workload's shapes)",
        "config": {"workload": WORKLOAD, "tokens": W.TOKENS, "linears": [list(l[1:]) for l in W.LINEARS],
                   "gemm_gflop_per_step": round(stack.flops / 1e9, 2),
                   "quant_elems_per_step": stack.q_elems,
                   "l2": f"{N_SETS} rotating input sets ({N_SETS * 2 * stack.q_elems / 1e6:.0f} MB bf16) > 126 MB L2",
                   "launch": ("CUDA graph per step" if used_graphs else "eager") +
                             (", dX + dW of each linear in one grouped GEMM launch" if stack.use_group_bwd() else
                              ", 1 stream" if side is None else
                              ", 2 streams (dX||dW" + (")" if grouped else ", x||W quantize)")) +
                             (", all W + first x quantized in one grouped launch" if grouped else "") +
                             (f", GEMMs split {stack.split_k} ways along K" if stack.split_k > 1 else "") +
                             (", data-parallel amax all-reduce + one ring fold per step" if stack.dp_amax else ""),
                   "launches_per_step": stack.launches_per_step(grouped),
                   "order": "forward over linears, then backward in reverse",
                   "parallelism": f"replicas x{world}" + (" with the amax all-reduce" if stack.dp_amax else "")},
        "quantize_gbs": round(quant_gbs, 1),
        "roofline": {"bound": "tensor", "achieved": round(gemm_tf, 1), "peak": round(fp8_burst, 1),
                     "unit": "TFLOP/s", "frac": round(gemm_tf / fp8_burst, 4),
                     "traffic": measured_traffic("gemm"),
                     "kernel": "fp8_gemm_kernel (all GEMM launches of a step, FLOP-weighted: "
                               + ("4 forward + 4 grouped dX+dW)" if stack.use_group_bwd() else "12 single GEMMs)"),
                     "peak_source": f"{peak_src}: 2 x bf16 burst {bf16_burst} TF/s (nominal fp8:bf16 = 2)",
                     "algorithmic_bytes_per_launch": round(g_bytes / n_g),
                     "flops_per_launch": round(g_flops / n_g),
                     "avg_launch_us": round(1e3 * g_ms / n_g, 2)},
        "roofline_quantize": {"bound": "hbm", "achieved": round(quant_gbs, 1), "peak": hbm, "unit": "GB/s",
                              "frac": round(quant_gbs / hbm, 4), "traffic": measured_traffic("quantize"),
                              "kernel": "quantize_kernel, delayed, each of the step's 12 tensors in a launch of "
                                        "its own (the step runs one grouped launch for every W and the first x, "
                                        "then 7 of these)",
                              "peak_source": f"{peak_src} hbm copy",
                              "algorithmic_bytes_per_launch": round(3 * q_elems / n_q),
                              "avg_launch_us": round(1e3 * q_ms / n_q, 2)},
        "breakdown_method": "each kernel repeated back to back, inputs and outputs rotating over copies that "
                            "exceed 2x L2 (HBM reads, as in the step); us_l2_hot: the same on one set",
        "gemm_by_shape": gemm_detail,
        "quantize_by_tensor": quant_detail,
        "kernels_l2_hot": l2_hot,
        "quantize_grouped": grouped_detail,
        "configs": configs,
        "clocks": clocks.summary(),
        "context": context,
        "e2e": e2e,
        "gpu_launches": gpu_launches,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_full_step()
    if rank == 0:
        print(json.dumps(line), flush=True)


def _rotated_graph_time(make_fn, reps, warm=3, n_sets=N_SETS):
    """One CUDA graph per input set, replayed in rotation over the sets, as
    the FP8 step is timed; ms per replay."""
    st = torch.cuda.Stream()
    fns = [make_fn(s) for s in range(n_sets)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(warm):
            for f in fns:
                f()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graphs = []
    for f in fns:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            f()
        graphs.append(g)
    torch.cuda.synchronize()
    with torch.cuda.stream(st):
        for i in range(warm * n_sets):
            graphs[i % n_sets].replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for i in range(reps):
            graphs[i % n_sets].replay()
        e1.record(st)
    e1.synchronize()
    ms = e0.elapsed_time(e1) / reps
    graphs.clear()
    return ms


def compare_bf16(stack, fp8_ms, reps):
    """The same linear-stack training step with bf16 GEMMs on cuBLAS
    (torch.matmul: forward, then dX and dW in reverse, one stream, which
    measured faster than putting dW on a second stream), and the step
    through the autograd layer (Fp8Linear against bf16 nn.Linear). Each is
    timed like the FP8 step: CUDA graphs over the same 3 rotating input sets
    (the autograd modules keep one weight each, as in training). Context
    for the FP8-over-bf16 speed-up the AstrAI commit logs report for their
    kernels on L20."""
    out = {}
    T = stack.tokens
    n_sets = len(stack.sets)
    ys = [torch.empty(T, L["d_out"], dtype=torch.bfloat16, device="cuda") for L in stack.lin]
    dxs = [torch.empty(T, L["d_in"], dtype=torch.bfloat16, device="cuda") for L in stack.lin]
    dws = [torch.empty(L["d_out"], L["d_in"], dtype=torch.bfloat16, device="cuda") for L in stack.lin]

    def bf16_step(s):
        ts = stack.sets[s]

        def fn():
            for li, t in enumerate(ts):
                torch.matmul(t["x"], t["w"].t(), out=ys[li])
            for li in reversed(range(len(ts))):
                t = ts[li]
                torch.matmul(t["g"], t["w"], out=dxs[li])
                torch.matmul(t["g"].t(), t["x"], out=dws[li])
        return fn

    bf16_ms = _rotated_graph_time(bf16_step, reps, n_sets=n_sets)
    out["bf16_cublas_step_ms"] = round(bf16_ms, 4)
    out["fp8_over_bf16_step"] = round(bf16_ms / fp8_ms, 3)

    # through torch.autograd: Fp8Linear vs bf16 nn.Linear, forward + backward
    try:
        from fp8_delayed_scaling_quantize_b200.linear import Fp8Linear
        mods8 = [Fp8Linear(L["d_in"], L["d_out"], bias=False, device="cuda") for L in stack.lin]
        mods16 = [torch.nn.Linear(L["d_in"], L["d_out"], bias=False, device="cuda", dtype=torch.bfloat16)
                  for L in stack.lin]
        xs = [[t["x"].detach().clone().requires_grad_(True) for t in stack.sets[s]] for s in range(n_sets)]

        def ag_step(mods):
            def make(s):
                def fn():
                    for m in mods:
                        m.weight.grad = None
                    for x in xs[s]:
                        x.grad = None
                    ys_ = [m(x) for m, x in zip(mods, xs[s])]
                    torch.autograd.backward(ys_, [t["g"] for t in stack.sets[s]])
                return fn
            return make

        out["autograd_fp8_step_ms"] = round(_rotated_graph_time(ag_step(mods8), reps, n_sets=n_sets), 4)
        out["autograd_bf16_step_ms"] = round(_rotated_graph_time(ag_step(mods16), reps, n_sets=n_sets), 4)
        out["autograd_fp8_over_bf16"] = round(out["autograd_bf16_step_ms"] / out["autograd_fp8_step_ms"], 3)
    except Exception as e:  # capture failures are reported, not hidden
        out["autograd_error"] = f"{type(e).__name__}: {e}"[:200]
    return out


def compare_at_tokens(fp8, tokens, reps):
    """The FP8 step and its bf16 / autograd comparisons at a larger token
    count: one input set (more than 2x L2 at 16384 tokens), the step as one
    CUDA graph."""
    stack = Stack(fp8, n_sets=1, tokens=tokens)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        for _ in range(3):
            stack.step(0, st, None, True)
    torch.cuda.synchronize()
    ms = _rotated_graph_time(lambda s: (lambda: stack.step(0, torch.cuda.current_stream(), None, True)), reps,
                             n_sets=1)
    out = {"tokens": tokens, "fp8_step_ms": round(ms, 4), "fp8_step_tflops": round(stack.flops / (ms * 1e-3) / 1e12, 1)}
    out.update(compare_bf16(stack, ms, reps))
    del stack
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_e2e(fp8, stack, stream, steps, world, side=None, grouped=True):
    """H2D of the step's inputs from pinned host memory, the step's calls, D2H of
    the three GEMM outputs, every step; CUDA events around the whole loop.

    The copies are pipelined as a training input pipeline would be: inputs
    and outputs are double-buffered on the device, host-to-device copies run
    on one copy stream and device-to-host copies on another (PCIe is full
    duplex), so step i's outputs leave while step i+1's inputs arrive. Every
    step still moves all of its bytes both ways inside the timed region."""
    host_in = [{k: v.cpu().pin_memory() for k, v in t.items()} for t in stack.sets[0]]
    outs = [[{k: L[k] for k in ("y", "dx", "dw")} for L in stack.lin],
            [{k: torch.empty_like(L[k]) for k in ("y", "dx", "dw")} for L in stack.lin]]
    host_out = [[{k: torch.empty(L[k].numel(), dtype=torch.bfloat16).pin_memory() for k in ("y", "dx", "dw")}
                 for L in stack.lin] for _ in range(2)]
    h2d = sum(v.numel() * 2 for t in host_in for v in t.values())
    d2h = sum(v.numel() * 2 for t in host_out[0] for v in t.values())
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("in", "used", "out", "sent")}
    for k in ("used", "sent"):
        for e in ev[k]:
            e.record(stream)

    def one(i):
        p = i % 2  # input set p and output buffers p
        up.wait_event(ev["used"][p])          # step i-2 has finished reading set p
        with torch.cuda.stream(up):
            for li, t in enumerate(host_in):
                for k, v in t.items():
                    stack.sets[p][li][k].copy_(v, non_blocking=True)
        ev["in"][p].record(up)
        stream.wait_event(ev["in"][p])
        stream.wait_event(ev["sent"][p])      # step i-2's outputs p have left
        for L, o in zip(stack.lin, outs[p]):
            L.update(o)
        stack.step(p, stream, side, grouped)
        ev["used"][p].record(stream)
        down.wait_event(ev["used"][p])
        with torch.cuda.stream(down):
            for li, L in enumerate(outs[p]):
                for k in ("y", "dx", "dw"):
                    host_out[p][li][k].copy_(L[k], non_blocking=True)
        ev["sent"][p].record(down)

    for i in range(2):
        one(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        one(i)
    stream.wait_stream(up)
    stream.wait_stream(down)
    e1.record(stream)
    e1.synchronize()
    barrier(world)
    for L, o in zip(stack.lin, outs[0]):
        L.update(o)
    t_ms = max_over_ranks(e0.elapsed_time(e1), world)
    return {"value": weak_scaling_value(stack.flops, steps, world, t_ms), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(t_ms / steps, 3),
            "pipeline": "inputs and outputs double-buffered; H2D and D2H on two copy streams"}


# ------------------------------------------------- the other workloads -----
#
# The workload table's other configurations, timed in the same run under the
# same clock record: the NT 256^3 GEMM with bias, the square sweep in all
# three layouts, the skinny shapes with bias, the batched shapes, and the
# quantize size sweep. Every timed loop runs back to back on one stream held
# in a device sleep while the host enqueues, and rotates over enough distinct
# buffer sets that one pass over them is more than twice the L2, so every
# launch reads its operands from HBM (the 256^3 case is 0.3 MB and stays
# L2-resident: it is latency-bound and reported in microseconds).

def _l2_bytes():
    try:
        return int(torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size)
    except Exception:
        return 126 << 20


def _slots(set_bytes, cap=64):
    """Buffer sets so that one rotation moves more than twice the L2."""
    return int(min(cap, max(2, -(-2 * _l2_bytes() // max(1, set_bytes)))))


def _time_us(stream, call, reps, warm=3):
    """Device microseconds per call of call(i), i = 0 .. reps-1, back to back."""
    with torch.cuda.stream(stream):
        for i in range(warm):
            call(i)
    torch.cuda.synchronize()
    hold_stream(stream, 500 + 40 * reps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(reps):
            call(warm + i)  # the rotation continues where the warm-up left it
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) * 1e3 / reps


def _gemm_entry(us, flops, nbytes, hbm, fp8_peak):
    """One GEMM's line: time, TF/s and its fraction of the binding roof
    (the slower of FLOPs at the FP8 peak and compulsory bytes at HBM)."""
    t_tensor = flops / (fp8_peak * 1e12) * 1e6
    t_hbm = nbytes / (hbm * 1e9) * 1e6
    bound = "tensor" if t_tensor >= t_hbm else "hbm"
    return {"us": round(us, 2), "tflops": round(flops / (us * 1e-6) / 1e12, 1),
            "gbs": round(nbytes / (us * 1e-6) / 1e9, 1), "bound": bound,
            "frac": round(max(t_tensor, t_hbm) / us, 4)}


def run_configs(fp8, stream, hbm, fp8_peak, reps=20):
    """Every workload of the table but the linear stack, timed on the device."""
    dev = "cuda"
    out = {"method": "back-to-back launches, CUDA events on the launching stream; buffers rotate over sets "
                     "whose total is > 2x L2, so operands come from HBM (except the 0.3 MB NT 256^3)"}

    def ring():
        r = torch.empty(20, dtype=torch.int32, device=dev)
        fp8.fp8_ring_init(r, 1.0)
        return r

    one = lambda v: torch.tensor([float(v)], device=dev)

    # -- NT 256^3, A and B current-scaled to E4M3 from bf16, bf16 bias --------
    M = N = K = 256
    a = W.bf16_normal((M, K), 1.0, 1001).to(dev)
    b = W.bf16_normal((N, K), 1.0, 1002).to(dev)
    bias = W.bf16_normal((N,), 0.1, 1003).to(dev)
    a8 = torch.empty(M * K, dtype=torch.uint8, device=dev)
    b8 = torch.empty(N * K, dtype=torch.uint8, device=dev)
    am, bm, sa, sb = (torch.empty(1, device=dev) for _ in range(4))
    y = torch.empty(M * N, dtype=torch.bfloat16, device=dev)
    qa = lambda i: fp8.fp8_quantize(a, M * K, E4M3, None, a8, am, sa, stream=stream)
    qb = lambda i: fp8.fp8_quantize(b, N * K, E4M3, None, b8, bm, sb, stream=stream)
    mm = lambda i: fp8.fp8_mm(a8, E4M3, b8, E4M3, sa, sb, NT, M, N, K, 1, 0, 0, 0, bias, None, 0, y, stream=stream)

    qab = lambda i: fp8.fp8_quantize_current_many([(a, M * K, E4M3, None, a8, am, sa), (b, N * K, E4M3, None, b8, bm, sb)],
                                                  stream=stream)

    def seq(i):
        qa(i)
        qb(i)
        mm(i)

    def seq_grouped(i):
        qab(i)
        mm(i)
    out["nt_256_bias_current"] = {
        "us_quantize_a": round(_time_us(stream, qa, reps), 2), "us_gemm": round(_time_us(stream, mm, reps), 2),
        "us_sequence": round(_time_us(stream, seq, reps), 2),
        "us_quantize_a_and_b_one_launch": round(_time_us(stream, qab, reps), 2),
        "us_sequence_grouped": round(_time_us(stream, seq_grouped, reps), 2),
        "bound": "latency (0.03 GFLOP, 0.3 MB)",
        "sequence": "current-scaled quantize of A and of B (one single-block launch each), GEMM + bias; "
                    "grouped: A and B current-scaled in one launch (fp8_quantize_current_many), GEMM + bias"}

    # -- square sweep on pre-quantized codes, NT / NN / TN ---------------------
    sq = {}
    for n in W.SQUARE_SIZES:
        set_bytes = 2 * n * n + 2 * n * n
        k = _slots(set_bytes)
        ha = W.fp8_codes((n * n,), E4M3, 3000 + n)
        hb = W.fp8_codes((n * n,), E4M3, 3100 + n)
        sc = W.uniform(0.5, 2.0, 3200 + n, 2)
        A = [ha.to(dev) for _ in range(k)]
        B = [hb.to(dev) for _ in range(k)]
        C = [torch.empty(n * n, dtype=torch.bfloat16, device=dev) for _ in range(k)]
        s_a, s_b = one(sc[0]), one(sc[1])
        r = 10 if n >= 8192 else reps
        for lay, name in ((NT, "NT"), (NN, "NN"), (TN, "TN")):
            call = lambda i, lay=lay: fp8.fp8_mm(A[i % k], E4M3, B[i % k], E4M3, s_a, s_b, lay, n, n, n, 1, 0, 0, 0,
                                                  None, None, 0, C[i % k], stream=stream)
            us = _time_us(stream, call, r)
            e = _gemm_entry(us, 2.0 * n ** 3, gemm_algorithmic_bytes(lay, n, n, n), hbm, fp8_peak)
            e["sets"] = k
            sq[f"{name} {n}^3"] = e
        del A, B, C
    out["square"] = sq

    # -- skinny / rectangular NT with bf16 bias, current-scaled operands -------
    sk = {}
    for (M, N, K) in W.SKINNY_SHAPES:
        set_bytes = M * K + N * K + 2 * M * N
        k = _slots(set_bytes)
        xa = W.bf16_normal((M * K,), 1.0, 4000 + M).to(dev)
        xb = W.bf16_normal((N * K,), 1.0, 4100 + N + K).to(dev)
        bias = W.bf16_normal((N,), 0.1, 4200 + N).to(dev)
        a8 = torch.empty(M * K, dtype=torch.uint8, device=dev)
        b8 = torch.empty(N * K, dtype=torch.uint8, device=dev)
        am, bm, s_a, s_b = (torch.empty(1, device=dev) for _ in range(4))
        fp8.fp8_quantize(xa, M * K, E4M3, None, a8, am, s_a, stream=stream)
        us_qb = _time_us(stream, lambda i: fp8.fp8_quantize(xb, N * K, E4M3, None, b8, bm, s_b, stream=stream), reps)
        A = [a8.clone() for _ in range(k)]
        B = [b8.clone() for _ in range(k)]
        C = [torch.empty(M * N, dtype=torch.bfloat16, device=dev) for _ in range(k)]
        call = lambda i: fp8.fp8_mm(A[i % k], E4M3, B[i % k], E4M3, s_a, s_b, NT, M, N, K, 1, 0, 0, 0, bias, None,
                                     0, C[i % k], stream=stream)
        us = _time_us(stream, call, reps)
        e = _gemm_entry(us, 2.0 * M * N * K, gemm_algorithmic_bytes(NT, M, N, K) + 2 * N, hbm, fp8_peak)
        e["sets"] = k
        e["us_quantize_b_current"] = round(us_qb, 2)
        sk[f"NT {M}x{N}x{K} +bias"] = e
        del A, B, C
    out["skinny"] = sk

    # -- batched, per-tensor scales; the second case broadcasts B ---------------
    bt = {}
    for (batch, M, N, K, bcast) in W.BATCHED:
        nb = 1 if bcast else batch
        set_bytes = batch * M * K + nb * N * K + 2 * batch * M * N
        k = _slots(set_bytes)
        ha = W.fp8_codes((batch * M * K,), E4M3, 5000 + batch)
        hb = W.fp8_codes((nb * N * K,), E4M3, 5100 + batch)
        A = [ha.to(dev) for _ in range(k)]
        B = [hb.to(dev) for _ in range(k)]
        C = [torch.empty(batch * M * N, dtype=torch.bfloat16, device=dev) for _ in range(k)]
        s_a, s_b = one(0.75), one(1.5)
        sbt = 0 if bcast else N * K
        call = lambda i: fp8.fp8_mm(A[i % k], E4M3, B[i % k], E4M3, s_a, s_b, NT, M, N, K, batch, M * K, sbt, M * N,
                                     None, None, 0, C[i % k], stream=stream)
        us = _time_us(stream, call, reps)
        e = _gemm_entry(us, 2.0 * batch * M * N * K, set_bytes, hbm, fp8_peak)
        e["sets"] = k
        bt[f"{batch}x{M}x{N}x{K}" + (" B stride 0" if bcast else "")] = e
        del A, B, C
    out["batched"] = bt

    # -- quantize sweep: delayed E4M3, 3 B per element --------------------------
    qs = {}
    base = W.bf16_normal((1 << 24,), 1.0, 6001).to(dev)
    for lg in (22, 24, 26, 28):
        n = 1 << lg
        k = _slots(3 * n)
        reps_q = max(reps, k)
        X = [base[:n].clone() if n <= base.numel() else base.repeat(n // base.numel()) for _ in range(k)]
        Q = [torch.empty(n, dtype=torch.uint8, device=dev) for _ in range(k)]
        rg = ring()
        am, sc = torch.empty(1, device=dev), torch.empty(1, device=dev)
        call = lambda i: fp8.fp8_quantize(X[i % k], n, E4M3, rg, Q[i % k], am, sc, stream=stream)
        us = _time_us(stream, call, reps_q)
        gbs = 3.0 * n / (us * 1e-6) / 1e9
        qs[f"2^{lg}"] = {"us": round(us, 2), "gbs": round(gbs, 1), "frac": round(gbs / hbm, 4), "sets": k}
        del X, Q
    out["quantize_delayed_e4m3"] = qs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------- the CPU oracle -----

def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return 1


def oracle_prepare(step_tensors):
    """Untimed set-up for the oracle legs: bf16 inputs as fp32 arrays, their
    codes and scales (one delayed step each), so that timed samples of the
    GEMMs run on the step's real operands."""
    import oracle
    prep = []
    for (_, d_in, d_out), t in zip(W.LINEARS, step_tensors):
        P = {"d_in": d_in, "d_out": d_out, "f": {}, "q": {}, "s": {}}
        for r, fmt in (("x", E4M3), ("w", E4M3), ("g", E5M2)):
            P["f"][r] = t[r].reshape(-1).float().numpy()
            ring = oracle.DelayedRing()
            ring.step(P["f"][r], fmt)
            P["q"][r], _, P["s"][r] = ring.step(P["f"][r], fmt)
        prep.append(P)
    return prep


def oracle_sample_step(prep, frac=1, blk=1):
    """One step of the oracle on a sample of the workload: the first 1/frac
    of every quantize input (a delayed ring step) and, of every GEMM, the
    leading (M/blk) x (N/blk) block of outputs with full K (the oracle called
    on the operand slices that block needs). frac = blk = 1 is the whole
    step. Returns (seconds, GEMM FLOPs computed, elements quantized)."""
    import oracle
    T = W.TOKENS
    flops = elems = 0
    t0 = time.perf_counter()
    for P in prep:
        for r, fmt in (("x", E4M3), ("w", E4M3), ("g", E5M2)):
            x = P["f"][r]
            n = x.size if frac == 1 else max(16, x.size // frac)
            oracle.DelayedRing().step(x[:n], fmt)
            elems += n
        d_in, d_out, q, s = P["d_in"], P["d_out"], P["q"], P["s"]
        xq = q["x"].reshape(T, d_in)
        wq = q["w"].reshape(d_out, d_in)
        gq = q["g"].reshape(T, d_out)
        m, n_out, n_in, m_dw = T // blk, d_out // blk, d_in // blk, d_out // blk
        # forward NT: rows of x, rows of W
        oracle.mm(xq[:m].reshape(-1), E4M3, wq[:n_out].reshape(-1), E4M3, s["x"], s["w"], oracle.NT,
                  m, n_out, d_in)
        # dX NN: rows of g, columns of W ([K = d_out, N = d_in])
        oracle.mm(gq[:m].reshape(-1), E5M2, np.ascontiguousarray(wq[:, :n_in]).reshape(-1), E4M3,
                  s["g"], s["w"], oracle.NN, m, n_in, d_out)
        # dW TN: columns of g ([K = T, M = d_out]), columns of x ([K = T, N = d_in])
        oracle.mm(np.ascontiguousarray(gq[:, :m_dw]).reshape(-1), E5M2,
                  np.ascontiguousarray(xq[:, :n_in]).reshape(-1), E4M3, s["g"], s["x"], oracle.TN,
                  m_dw, n_in, T)
        flops += 2 * m * n_out * d_in + 2 * m * n_in * d_out + 2 * m_dw * n_in * T
    return time.perf_counter() - t0, flops, elems


def cpu_baseline_full_step():
    """The oracle as it stands on one full step of the workload (rank 0), on
    all the host's BLAS threads; beside it the same oracle held to one thread
    on a 1/16 sample of the step."""
    prep = oracle_prepare(W.stack_tensors(0))
    dt, flops, elems = oracle_sample_step(prep)
    out = {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
           "sample": f"one full step: 12 delayed quantizes ({elems / 1e6:.1f} M elements) + 12 fp64 GEMMs "
                     f"({flops / 1e9:.1f} GFLOP)", "seconds": round(dt, 2)}
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        return out
    with threadpool_limits(limits=1):
        dt1, f1, e1 = oracle_sample_step(prep, 16, 4)
    out["single_thread"] = {"value": round(f1 / dt1 / 1e12, 6), "unit": "TFLOP/s", "cores": 1,
                            "sample": f"1/16 of the step: the first 1/16 of each quantize input ({e1 / 1e6:.1f} M "
                                      f"elements) and an (M/4) x (N/4) output block of each GEMM "
                                      f"({f1 / 1e9:.1f} GFLOP)", "seconds": round(dt1, 2)}
    return out


REF_FRAC, REF_BLK = 256, 16


def run_reference(args, world, rank):
    """The oracle on the host cores; each bench step is a bounded sample of
    the stack step: 1/256 of every quantize input and a (M/16) x (N/16)
    output block of every GEMM (1/256 of its FLOPs)."""
    if rank != 0:
        return
    prep = oracle_prepare(W.stack_tensors(0))
    for _ in range(args.warmup):
        oracle_sample_step(prep, REF_FRAC, REF_BLK)
    total = flops = 0
    for _ in range(args.steps):
        dt, f, _ = oracle_sample_step(prep, REF_FRAC, REF_BLK)
        total += dt
        flops += f
    v = flops / total / 1e12
    sample = (f"per step: the first 1/{REF_FRAC} of each of the 12 quantize inputs and a (M/{REF_BLK}) x "
              f"(N/{REF_BLK}) output block, full K, of each of the 12 GEMMs ({flops / args.steps / 1e9:.3f} GFLOP)")
    line = {"metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle: fp32 quantize, fp64 GEMM)",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_kernel(args):
    """Single-kernel mode (profiling and sweeps): one GEMM shape or one
    quantize size, repeated; prints per-launch device time and roofline."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    hbm, bf16_burst, _, src = _peaks()
    st = torch.cuda.Stream()
    reps = max(args.steps, 1)
    if args.kernel == "cublaslt":
        # in-box comparison: cuBLASLt's FP8 GEMM through torch._scaled_mm on
        # the same NT problem (A [M,K] row-major, B [N,K] row-major = a
        # column-major [K,N] operand); scales are its dequantisation factors
        M, N, K = (int(v) for v in args.shape.split("x"))
        sets = []
        for i in range(2):
            a = W.fp8_codes((M, K), E4M3, 9100 + i).cuda().view(torch.float8_e4m3fn)
            b = W.fp8_codes((N, K), E4M3, 9200 + i).cuda().view(torch.float8_e4m3fn)
            sets.append((a, b))
        one = torch.ones((), device="cuda")
        call = lambda i: torch._scaled_mm(sets[i % 2][0], sets[i % 2][1].t(), scale_a=one, scale_b=one,
                                          out_dtype=torch.bfloat16)
        units = 2.0 * M * N * K
    elif args.kernel == "gemm":
        M, N, K = (int(v) for v in args.shape.split("x"))
        layout = {"NT": NT, "NN": NN, "TN": TN}[args.layout]
        sets = []
        for i in range(2):
            a = W.fp8_codes((M * K,), E4M3, 9100 + i).cuda()
            b = W.fp8_codes((N * K,), E4M3, 9200 + i).cuda()
            sets.append((a, b))
        sa = torch.ones(1, device="cuda")
        out = torch.empty(M * N, dtype=torch.bfloat16, device="cuda")
        need = fp8.fp8_mm_workspace_size(M, N, K, 1, layout, args.split_k)
        ws = torch.zeros(max(need, 4096), dtype=torch.uint8, device="cuda") if need else None
        call = lambda i: fp8.fp8_mm_ws(sets[i % 2][0], E4M3, sets[i % 2][1], E4M3, sa, sa, layout, M, N, K, 1, 0, 0,
                                       0, None, None, 0, out, ws, args.split_k if need else 0, stream=st)
        units = 2.0 * M * N * K
    elif args.kernel == "bwd_pair":
        # a linear's backward as the step runs it: dX = g W (NN) and
        # dW = g^T x (TN) in one grouped launch; --shape T x d_in x d_out
        T, d_in, d_out = (int(v) for v in args.shape.split("x"))
        sets = []
        for i in range(2):
            g8 = W.fp8_codes((T * d_out,), E5M2, 9600 + i).cuda()
            w8 = W.fp8_codes((d_out * d_in,), E4M3, 9700 + i).cuda()
            x8 = W.fp8_codes((T * d_in,), E4M3, 9800 + i).cuda()
            sets.append((g8, w8, x8))
        sa = torch.ones(1, device="cuda")
        dx = torch.empty(T * d_in, dtype=torch.bfloat16, device="cuda")
        dw = torch.empty(d_out * d_in, dtype=torch.bfloat16, device="cuda")
        call = lambda i: fp8.fp8_mm_grouped(
            [(sets[i % 2][0], E5M2, sets[i % 2][1], E4M3, sa, sa, NN, T, d_in, d_out, None, None, 0, dx),
             (sets[i % 2][0], E5M2, sets[i % 2][2], E4M3, sa, sa, TN, d_out, d_in, T, None, None, 0, dw)], stream=st)
        units = 2.0 * 2 * T * d_in * d_out
    elif args.kernel == "quantize_2d":
        # both orientations of a bf16 [rows, cols] tensor from one pass, delayed
        rows, cols = (int(v) for v in args.shape.split("x"))
        xs = [W.bf16_normal((rows, cols), 1.0, 9500 + i).cuda() for i in range(2)]
        q = torch.empty(rows * cols, dtype=torch.uint8, device="cuda")
        qt = torch.empty(rows * cols, dtype=torch.uint8, device="cuda")
        ring = torch.empty(20, dtype=torch.int32, device="cuda")
        fp8.fp8_ring_init(ring, 1.0)
        sc = torch.empty(1, device="cuda")
        am = torch.empty(1, device="cuda")
        call = lambda i: fp8.fp8_quantize_2d(xs[i % 2], 0, rows, cols, E4M3, ring, 0, 2, q, qt, am, sc, stream=st)
        units = 4.0 * rows * cols  # 2 bytes read, 1 + 1 written per element
    elif args.kernel == "quantize_many":
        # the linear stack's step-start launch: every weight and the first x
        sizes = [d_out * d_in for _, d_in, d_out in W.LINEARS] + [W.TOKENS * W.LINEARS[0][1]]
        xs = [[W.bf16_normal((n,), 1.0, 9400 + 10 * i + j).cuda() for j, n in enumerate(sizes)] for i in range(2)]
        qs = [torch.empty(n, dtype=torch.uint8, device="cuda") for n in sizes]
        rings = [torch.empty(20, dtype=torch.int32, device="cuda") for _ in sizes]
        for r in rings:
            fp8.fp8_ring_init(r, 1.0)
        scs = [torch.empty(1, device="cuda") for _ in sizes]
        ams = [torch.empty(1, device="cuda") for _ in sizes]
        jobs = [[(xs[i][j], n, E4M3, rings[j], qs[j], ams[j], scs[j]) for j, n in enumerate(sizes)] for i in range(2)]
        call = lambda i: fp8.fp8_quantize_many(jobs[i % 2], stream=st)
        units = 3.0 * sum(sizes)
    else:
        n = int(args.shape)
        xs = [W.bf16_normal((n,), 1.0, 9300 + i).cuda() for i in range(2)]
        q = torch.empty(n, dtype=torch.uint8, device="cuda")
        ring = torch.empty(20, dtype=torch.int32, device="cuda")
        fp8.fp8_ring_init(ring, 1.0)
        sc = torch.empty(1, device="cuda")
        am = torch.empty(1, device="cuda")
        call = lambda i: fp8.fp8_quantize(xs[i % 2], n, E4M3, ring, q, am, sc, stream=st)
        units = 3.0 * n
    with torch.cuda.stream(st):
        for i in range(max(args.warmup, 3)):
            call(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        # the hold starts after the sampler's set-up, so it still covers the
        # host's enqueueing of every timed launch
        hold_stream(st, 2000 + 40 * reps)
        with torch.cuda.stream(st):
            e0.record(st)
            for i in range(reps):
                call(i)
            e1.record(st)
        torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    if args.kernel in ("gemm", "cublaslt", "bwd_pair"):
        ach = units / (us * 1e-6) / 1e12
        peak = 2 * bf16_burst
        print(json.dumps({"kernel": args.kernel, "shape": args.shape,
                          "layout": {"gemm": args.layout, "cublaslt": "NT", "bwd_pair": "NN + TN"}[args.kernel],
                          "us": round(us, 2),
                          "tflops": round(ach, 1), "frac_fp8_peak": round(ach / peak, 4), "peak": peak,
                          "peak_source": src, "clocks": clocks.summary()}))
    else:
        ach = units / (us * 1e-6) / 1e9
        n_el = int(units / 4) if args.kernel == "quantize_2d" else int(units / 3)
        print(json.dumps({"kernel": args.kernel, "n": n_el, "us": round(us, 2), "gbs": round(ach, 1),
                          "frac_hbm": round(ach / hbm, 4), "peak": hbm, "peak_source": src,
                          "clocks": clocks.summary()}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--one-stream", action="store_true", help="issue the whole step on one stream")
    ap.add_argument("--no-grouped", action="store_true", help="quantize every tensor with its own launch")
    ap.add_argument("--no-group-bwd", action="store_true",
                    help="run each linear's dX and dW as two GEMM launches (two streams) instead of one grouped launch")
    ap.add_argument("--split-k", type=int, default=0, help="force this many K splits in the GEMMs (0: library choice)")
    ap.add_argument("--dp-amax", action="store_true",
                    help="deferred ring folds + the ranks' amax all-reduce (MAX) and one fold per step")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-compare", action="store_true", help="skip the bf16 / autograd comparison")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (NT 256^3, square sweep, skinny, batched, quantize sweep)")
    ap.add_argument("--breakdown-reps", type=int, default=20)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--kernel", choices=["gemm", "bwd_pair", "quantize", "quantize_many", "quantize_2d", "cublaslt"],
                    help="single-kernel mode")
    ap.add_argument("--shape", default="8192x8192x8192", help="MxNxK for gemm, n for quantize")
    ap.add_argument("--layout", default="NT", choices=["NT", "NN", "TN"])
    args = ap.parse_args()
    if args.kernel:
        run_kernel(args)
        return
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
