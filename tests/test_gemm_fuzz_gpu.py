"""Seeded random GEMM problems against the oracle, in full.

Each seed draws one problem: layout, operand formats, M / N / K (the pitch
rules kept: K a multiple of 16 for K-major operands, M or N a multiple of 16
for MN-major ones; everything else free, odd sizes included), batches with
either operand broadcast, output padding between batches, bias kind and
scales. fp8_mm's output is held to the oracle's bar
|gpu - oracle| <= ulp_bf16(oracle) + 2^-16 * sum_k |a b| / (sa sb),
the padding must stay unwritten, and, where the problem can take it, a split
of K over a workspace is held to the same bar with its counters back at zero.
Groups of two or three drawn problems through fp8_mm_grouped are held to the
same bar, and equal fp8_mm bit for bit where fp8_mm does not swap operands.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import E4M3, E5M2, NN, NT, TN
import workloads as W

pytestmark = pytest.mark.gpu

MAX_MACS = 120_000_000  # keeps the oracle's fp64 products to a fraction of a second


@pytest.fixture(scope="module")
def g():
    import gpu_util
    return gpu_util


def _draw(rng, batch_ok=True):
    layout = int(rng.choice([NT, NN, TN]))
    fa, fb = (int(v) for v in rng.integers(0, 2, 2))

    def size(mult, small):
        if small:
            v = int(rng.integers(1, 41))
        else:
            v = int(rng.integers(16, 720))
        return max(mult, (v + mult - 1) // mult * mult) if mult > 1 else v

    small_m = rng.random() < 0.3
    M = size(16 if layout == TN else 1, small_m)
    N = size(16 if layout in (NN, TN) else 1, rng.random() < 0.15)
    K = size(1 if layout == TN else 16, rng.random() < 0.2)
    if layout == NT and small_m and rng.random() < 0.5:
        N = int(rng.integers(128, 1100))  # short problems with room to swap
        K = int(rng.integers(8, 160)) * 16
    batch = int(rng.choice([1, 1, 1, 2, 3])) if batch_ok else 1
    while M * N * K * batch > MAX_MACS:
        K = max(16, (K // 2 + 15) // 16 * 16) if layout != TN else max(1, K // 2)
        if K <= 16 and M * N * K * batch > MAX_MACS:
            batch = 1
            N = max(16, N // 2 // 16 * 16)
    bcast_a = batch > 1 and rng.random() < 0.3
    bcast_b = batch > 1 and not bcast_a and rng.random() < 0.4
    pad_c = int(rng.choice([0, 8, 3])) if batch > 1 else 0
    bias_kind = int(rng.integers(0, 3))
    sa = float(np.float32(rng.uniform(0.5, 2.0)))
    sb = float(np.float32(rng.uniform(0.5, 2.0)))
    return dict(layout=layout, fa=fa, fb=fb, M=M, N=N, K=K, batch=batch, bcast_a=bcast_a, bcast_b=bcast_b,
                pad_c=pad_c, bias_kind=bias_kind, sa=sa, sb=sb)


def _materialise(p, seed):
    M, N, K, batch = p["M"], p["N"], p["K"], p["batch"]
    p["a8"] = W.fp8_codes(((1 if p["bcast_a"] else batch) * M * K,), p["fa"], seed)
    p["b8"] = W.fp8_codes(((1 if p["bcast_b"] else batch) * N * K,), p["fb"], seed + 1)
    p["bias"] = p["bias_dev"] = p["bscale"] = p["bscale_dev"] = None
    if p["bias_kind"] == 1:
        b = W.bf16_normal((N,), 0.1, seed + 2)
        p["bias_dev"] = b.cuda()
        p["bias"] = b.view(torch.int16).numpy().view(np.uint16)
    elif p["bias_kind"] == 2:
        b = W.fp8_codes((N,), E5M2, seed + 2)
        p["bias"], p["bias_dev"] = b.numpy(), b.cuda()
        p["bscale"] = np.float32(4.0)
        p["bscale_dev"] = torch.tensor([p["bscale"]], device="cuda")
    p["stride_a"] = 0 if p["bcast_a"] else M * K
    p["stride_b"] = 0 if p["bcast_b"] else N * K
    p["stride_c"] = M * N + p["pad_c"]
    return p


def _oracle(p):
    return oracle.mm(p["a8"].numpy(), p["fa"], p["b8"].numpy(), p["fb"], p["sa"], p["sb"], p["layout"], p["M"],
                     p["N"], p["K"], batch=p["batch"], stride_a=p["stride_a"], stride_b=p["stride_b"],
                     bias=p["bias"], bias_scale=p["bscale"], bias_fmt=E5M2)


def _gpu(g, p, ws=None, split_k=0):
    sad = torch.tensor([p["sa"]], dtype=torch.float32, device="cuda")
    sbd = torch.tensor([p["sb"]], dtype=torch.float32, device="cuda")
    out = torch.full((p["batch"] * p["stride_c"] + 32,), float("nan"), dtype=torch.bfloat16, device="cuda")
    g.mm(p["a8"].cuda(), p["fa"], p["b8"].cuda(), p["fb"], sad, sbd, p["layout"], p["M"], p["N"], p["K"],
         batch=p["batch"], stride_a=p["stride_a"], stride_b=p["stride_b"], stride_c=p["stride_c"],
         bias=p["bias_dev"], bias_scale=p["bscale_dev"], bias_fmt=E5M2, out=out, ws=ws, split_k=split_k)
    return out


def _check(g, p, out, y, s, what):
    M, N, sc = p["M"], p["N"], p["stride_c"]
    got = out.float().cpu().numpy()
    res = np.stack([got[b * sc: b * sc + M * N].reshape(M, N) for b in range(p["batch"])])
    g.assert_within(res, y, oracle.tolerance(y, s), what)
    for b in range(p["batch"]):
        assert np.all(np.isnan(got[b * sc + M * N: (b + 1) * sc])), f"{what}: padding written"
    assert np.all(np.isnan(got[p["batch"] * sc:])), f"{what}: written past the end"


def _name(p):
    lay = {NT: "NT", NN: "NN", TN: "TN"}[p["layout"]]
    return (f"{lay} {p['M']}x{p['N']}x{p['K']} b{p['batch']} bcast({int(p['bcast_a'])},{int(p['bcast_b'])}) "
            f"pad{p['pad_c']} bias{p['bias_kind']} f({p['fa']},{p['fb']})")


@pytest.mark.parametrize("seed", range(160))
def test_random_problem(g, seed):
    import fp8_delayed_scaling_quantize_b200 as fp8
    rng = np.random.default_rng(31000 + seed)
    p = _materialise(_draw(rng), 32000 + 10 * seed)
    y, s = _oracle(p)
    _check(g, p, _gpu(g, p), y, s, _name(p))
    split = int(rng.integers(2, 5))
    need = fp8.fp8_mm_workspace_size(p["M"], p["N"], p["K"], p["batch"], p["layout"], split)
    if need > 4096:
        ws = g.workspace(need)
        try:
            out = _gpu(g, p, ws, split)
        except fp8.Fp8Error as e:
            assert e.status == fp8.FP8_ERR_UNSUPPORTED, e  # too few k-blocks for that split
        else:
            _check(g, p, out, y, s, _name(p) + f" split {split}")
            assert not ws[:4096].any(), "counters must be zero after the call"
    assert fp8.fp8_last_device_error() == fp8.FP8_OK


@pytest.mark.parametrize("seed", range(24))
def test_random_group(g, seed):
    import fp8_delayed_scaling_quantize_b200 as fp8
    rng = np.random.default_rng(33000 + seed)
    probs = [_materialise(_draw(rng, batch_ok=False), 34000 + 10 * (4 * seed + i))
             for i in range(int(rng.integers(2, 4)))]
    entries, outs, alone = [], [], []
    for p in probs:
        sad = torch.tensor([p["sa"]], dtype=torch.float32, device="cuda")
        sbd = torch.tensor([p["sb"]], dtype=torch.float32, device="cuda")
        a, b = p["a8"].cuda(), p["b8"].cuda()
        o = torch.full((p["M"] * p["N"],), float("nan"), dtype=torch.bfloat16, device="cuda")
        entries.append((a, p["fa"], b, p["fb"], sad, sbd, p["layout"], p["M"], p["N"], p["K"], p["bias_dev"],
                        p["bscale_dev"], E5M2, o))
        outs.append(o)
        alone.append(_gpu(g, p))
    fp8.fp8_mm_grouped(entries)
    torch.cuda.synchronize()
    for p, o, ref in zip(probs, outs, alone):
        y, s = _oracle(p)
        g.assert_within(o.float().cpu().numpy().reshape(1, p["M"], p["N"]), y, oracle.tolerance(y, s),
                        "group entry " + _name(p))
        # fp8_mm runs short problems (M <= 32, N >= 128, NT or NN) with swapped
        # operands, maybe split along K; every other problem takes the same
        # k-block order in both launches, so the same bits
        swapped = p["M"] <= 32 and p["N"] >= 128 and p["layout"] != TN
        if not swapped:
            assert torch.equal(o.view(torch.int16), ref[:p["M"] * p["N"]].view(torch.int16)), _name(p)
    assert fp8.fp8_last_device_error() == fp8.FP8_OK
