"""GPU parity of fp8_mm_grouped (several GEMMs in one launch) against the
CPU oracle, and its bit-for-bit agreement with fp8_mm on each problem.

Bar per problem: |gpu - oracle| <= ulp_bf16(oracle) + 2^-16 sum_k |a b| / (sa sb)
(oracle.tolerance). Small groups are compared in full, the linear stack's
backward pairs (dX NN + dW TN, one launch per layer) on sampled outputs.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import E4M3, E5M2, NN, NT, TN
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import gpu_util
    return gpu_util


def _dev(t):
    return t.contiguous().cuda()


def _shape(layout, M, N, K):
    return (M * K, N * K)


class Prob:
    """One problem: host codes, device copies, scales, optional bias, output."""

    def __init__(self, layout, M, N, K, fa, fb, seed, bias_kind=0, sa=0.75, sb=1.5):
        self.layout, self.M, self.N, self.K, self.fa, self.fb = layout, M, N, K, fa, fb
        self.a8 = W.fp8_codes((M * K,), fa, seed)
        self.b8 = W.fp8_codes((N * K,), fb, seed + 1)
        self.sa, self.sb = np.float32(sa), np.float32(sb)
        self.sad = torch.tensor([sa], dtype=torch.float32, device="cuda")
        self.sbd = torch.tensor([sb], dtype=torch.float32, device="cuda")
        self.bias = self.bias_dev = self.bscale = self.bscale_dev = None
        if bias_kind == 1:
            b = W.bf16_normal((N,), 0.1, seed + 2)
            self.bias_dev = _dev(b)
            self.bias = b.view(torch.int16).numpy().view(np.uint16)
        elif bias_kind == 2:
            b = W.fp8_codes((N,), E5M2, seed + 2)
            self.bias, self.bias_dev = b.numpy(), _dev(b)
            self.bscale = np.float32(5.0)
            self.bscale_dev = torch.tensor([self.bscale], device="cuda")
        self.a_dev, self.b_dev = _dev(self.a8), _dev(self.b8)
        # NaN guard after the output: nothing past M*N is written
        self.out = torch.full((M * N + 64,), float("nan"), dtype=torch.bfloat16, device="cuda")

    def tup(self):
        return (self.a_dev, self.fa, self.b_dev, self.fb, self.sad, self.sbd, self.layout, self.M, self.N,
                self.K, self.bias_dev, self.bscale_dev, E5M2, self.out)

    def single(self, g):
        return g.mm(self.a_dev, self.fa, self.b_dev, self.fb, self.sad, self.sbd, self.layout, self.M, self.N,
                    self.K, bias=self.bias_dev, bias_scale=self.bscale_dev, bias_fmt=E5M2)

    def check_full(self, g, what):
        y, s = oracle.mm(self.a8.numpy(), self.fa, self.b8.numpy(), self.fb, self.sa, self.sb, self.layout,
                         self.M, self.N, self.K, bias=self.bias, bias_scale=self.bscale, bias_fmt=E5M2)
        got = self.out.float().cpu().numpy()
        g.assert_within(got[:self.M * self.N].reshape(1, self.M, self.N), y, oracle.tolerance(y, s), what)
        assert np.all(np.isnan(got[self.M * self.N:])), what

    def check_same_as_fp8_mm(self, g, what):
        ref = self.single(g)
        torch.cuda.synchronize()
        assert torch.equal(self.out[:self.M * self.N].view(torch.int16), ref[:self.M * self.N].view(torch.int16)), what


def _run(probs):
    import fp8_delayed_scaling_quantize_b200 as fp8
    fp8.fp8_mm_grouped([p.tup() for p in probs])
    torch.cuda.synchronize()


GROUPS = [
    # layouts, formats, bias kinds and ragged edges mixed in one launch
    [(NN, 256, 384, 256, E5M2, E4M3, 0), (TN, 384, 256, 512, E5M2, E4M3, 0)],
    [(NT, 304, 272, 144, E4M3, E4M3, 1), (NN, 144, 144, 272, E4M3, E5M2, 2), (TN, 160, 96, 208, E5M2, E5M2, 0)],
    [(NT, 130, 20, 64, E4M3, E4M3, 0), (NT, 1, 7, 32, E4M3, E5M2, 1), (NN, 17, 48, 96, E5M2, E4M3, 2),
     (TN, 48, 80, 16, E4M3, E4M3, 1)],
    [(NT, 512, 1024, 640, E4M3, E4M3, 0)],
]


@pytest.mark.parametrize("gi", range(len(GROUPS)))
def test_grouped_small_full(g, gi):
    probs = [Prob(*spec[:6], seed=100 * gi + 10 * i, bias_kind=spec[6]) for i, spec in enumerate(GROUPS[gi])]
    _run(probs)
    for i, p in enumerate(probs):
        p.check_full(g, f"group {gi} problem {i}")
        p.check_same_as_fp8_mm(g, f"group {gi} problem {i} vs fp8_mm")


def test_grouped_many_tiles_unequal_k(g):
    """Four problems whose K differ, so the launch reorders them (longest K
    first) and unit ranges of all four meet inside one CTA's walk."""
    specs = [(NT, 640, 512, 256, E4M3, E4M3, 0), (NN, 512, 768, 1024, E5M2, E4M3, 0),
             (TN, 384, 512, 768, E5M2, E4M3, 1), (NT, 256, 1000, 128, E4M3, E5M2, 2)]
    probs = [Prob(*s[:6], seed=700 + 10 * i, bias_kind=s[6]) for i, s in enumerate(specs)]
    _run(probs)
    for i, p in enumerate(probs):
        p.check_full(g, f"unequal k problem {i}")
        p.check_same_as_fp8_mm(g, f"unequal k problem {i} vs fp8_mm")


def test_grouped_three_layouts_ragged_mid_size(g):
    """Three mid-size problems (several rounds of the persistent grid), ragged
    M and N, every layout, both bias kinds."""
    specs = [(NT, 1500, 1700, 512, E4M3, E4M3, 1), (NN, 1200, 1808, 256, E5M2, E4M3, 0),
             (TN, 704, 912, 640, E5M2, E4M3, 2)]
    probs = [Prob(*s[:6], seed=800 + 10 * i, bias_kind=s[6]) for i, s in enumerate(specs)]
    _run(probs)
    for i, p in enumerate(probs):
        p.check_full(g, f"mid-size problem {i}")
        p.check_same_as_fp8_mm(g, f"mid-size problem {i} vs fp8_mm")


def test_grouped_narrow_tail_ragged(g):
    """Two problems whose 128 x 256 tiles leave the grid's last round short:
    the launch runs the last problem's rightmost columns as 128-wide tiles
    (a second entry whose N edge is ragged). Full comparison with the oracle,
    with a bias on the split problem."""
    specs = [(NT, 2048, 1936, 384, E4M3, E4M3, 1), (NT, 1024, 1000, 640, E4M3, E5M2, 0)]
    probs = [Prob(*s[:6], seed=1700 + 10 * i, bias_kind=s[6]) for i, s in enumerate(specs)]
    _run(probs)
    for i, p in enumerate(probs):
        p.check_full(g, f"narrow tail problem {i}")
        p.check_same_as_fp8_mm(g, f"narrow tail problem {i} vs fp8_mm")


def test_fp8_mm_routed_through_narrow_tail(g):
    """fp8_mm of a shape whose last round of 128 x 256 tiles is short (QKV
    forward of the linear stack, and a ragged variant) runs as a grouped launch
    with a 128-wide tail; the output is compared in full with the oracle."""
    for spec in ((NT, 2048, 3072, 1024, E4M3, E4M3, 0), (NT, 1000, 3100, 512, E4M3, E4M3, 2)):
        p = Prob(*spec[:6], seed=1800, bias_kind=spec[6])
        out = p.single(g)
        torch.cuda.synchronize()
        p.out[:p.M * p.N].copy_(out[:p.M * p.N])
        p.check_full(g, f"routed fp8_mm {spec[:4]}")


def _sample_idx(M, N, seed):
    rng = np.random.default_rng(seed)
    i = rng.integers(0, M, 2048)
    j = rng.integers(0, N, 2048)
    rows = rng.integers(0, M, 4)
    i = np.concatenate([i, np.repeat(rows, N)])
    j = np.concatenate([j, np.tile(np.arange(N), 4)])
    return np.stack([np.zeros_like(i), i, j], axis=1)


def test_linear_stack_backward_pairs_sampled(g):
    """dX (NN) and dW (TN) of every linear of the stack in one launch each,
    at full size, on sampled outputs; both equal fp8_mm bit for bit."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    T = W.TOKENS
    for li, ((name, d_in, d_out), t) in enumerate(zip(W.LINEARS, W.stack_tensors(1))):
        qx, _, sxd = g.quantize(t["x"].reshape(-1).cuda(), E4M3, None)
        qw, _, swd = g.quantize(t["w"].reshape(-1).cuda(), E4M3, None)
        qg, _, sgd = g.quantize(t["g"].reshape(-1).cuda(), E5M2, None)
        dx = torch.empty(T * d_in, dtype=torch.bfloat16, device="cuda")
        dw = torch.empty(d_out * d_in, dtype=torch.bfloat16, device="cuda")
        fp8.fp8_mm_grouped([(qg, E5M2, qw, E4M3, sgd, swd, NN, T, d_in, d_out, None, None, 0, dx),
                            (qg, E5M2, qx, E4M3, sgd, sxd, TN, d_out, d_in, T, None, None, 0, dw)])
        torch.cuda.synchronize()
        sx, sw, sg = (float(g.f32(v)[0]) for v in (sxd, swd, sgd))
        for what, a8, fa, b8, fb, sa, sb, layout, M, N, K, out in (
                ("dX", qg, E5M2, qw, E4M3, sg, sw, NN, T, d_in, d_out, dx),
                ("dW", qg, E5M2, qx, E4M3, sg, sx, TN, d_out, d_in, T, dw)):
            idx = _sample_idx(M, N, 31 * li + len(what))
            y, s = oracle.mm_sampled(g.codes(a8), fa, g.codes(b8), fb, sa, sb, layout, M, N, K, idx)
            got = out.float().view(M, N)[torch.from_numpy(idx[:, 1]), torch.from_numpy(idx[:, 2])].cpu().numpy()
            g.assert_within(got, y, oracle.tolerance(y, s), f"{name} {what} grouped")
            ref = g.mm(a8, fa, b8, fb, sgd, sxd if what == "dW" else swd, layout, M, N, K)
            torch.cuda.synchronize()
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"{name} {what} vs fp8_mm"


def test_grouped_graph_replay(g):
    import fp8_delayed_scaling_quantize_b200 as fp8
    probs = [Prob(NN, 384, 256, 512, E5M2, E4M3, 900), Prob(TN, 256, 384, 384, E5M2, E4M3, 910, bias_kind=1)]
    _run(probs)
    first = [p.out.clone() for p in probs]
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        for p in probs:
            p.out.fill_(float("nan"))
        with torch.cuda.graph(graph, stream=s):
            fp8.fp8_mm_grouped([p.tup() for p in probs], stream=s)
    for _ in range(3):
        for p in probs:
            p.out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for p, f in zip(probs, first):
            assert torch.equal(p.out.view(torch.int16), f.view(torch.int16))
    del graph
    assert fp8.fp8_last_device_error() == fp8.FP8_OK
