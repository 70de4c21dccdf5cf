"""GPU parity of fp8_mm_ws, the GEMM that splits K over a workspace.

The split regroups the fp32 accumulation (per-split partial sums, then the
partials added in split order), so the bar is the same as fp8_mm's:
|gpu - oracle| <= ulp_bf16(oracle) + 2^-16 * sum_k |a b| / (sa sb) per output.
On top of it: the result is bit-identical from run to run and under CUDA-graph
replay (the partials are added in a fixed order whatever order the splits
finish in), the workspace's counters are zero after every call, a workspace
that is too small is refused, and split_k = 0 / 1 is fp8_mm bit for bit.
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


def _case(layout, M, N, K, fa, fb, seed, batch=1, bcast_b=False, bias_kind=0):
    bb = 1 if bcast_b else batch
    a8 = W.fp8_codes((batch * M * K,), fa, seed)
    b8 = W.fp8_codes((bb * N * K,), fb, seed + 1)
    bias = bias_dev = bscale = bscale_dev = None
    if bias_kind == 1:
        bb16 = W.bf16_normal((N,), 0.1, seed + 2)
        bias_dev = bb16.cuda()
        bias = bb16.view(torch.int16).numpy().view(np.uint16)
    elif bias_kind == 2:
        b = W.fp8_codes((N,), E5M2, seed + 2)
        bias, bias_dev = b.numpy(), b.cuda()
        bscale = np.float32(5.0)
        bscale_dev = torch.tensor([bscale], device="cuda")
    return dict(a8=a8, b8=b8, bias=bias, bias_dev=bias_dev, bscale=bscale, bscale_dev=bscale_dev,
                stride_b=0 if bcast_b else N * K)


def _run(g, c, layout, M, N, K, fa, fb, batch, ws, split_k=0, sa=0.75, sb=1.5):
    sad = torch.tensor([sa], dtype=torch.float32, device="cuda")
    sbd = torch.tensor([sb], dtype=torch.float32, device="cuda")
    out = torch.full((batch * M * N,), float("nan"), dtype=torch.bfloat16, device="cuda")
    g.mm(c["a8"].cuda(), fa, c["b8"].cuda(), fb, sad, sbd, layout, M, N, K, batch=batch,
         stride_b=c["stride_b"], bias=c["bias_dev"], bias_scale=c["bscale_dev"], bias_fmt=E5M2, out=out, ws=ws,
         split_k=split_k)
    return out


def _oracle(c, layout, M, N, K, fa, fb, batch, sa=0.75, sb=1.5):
    return oracle.mm(c["a8"].numpy(), fa, c["b8"].numpy(), fb, sa, sb, layout, M, N, K, batch=batch,
                     stride_a=M * K, stride_b=c["stride_b"], bias=c["bias"], bias_scale=c["bscale"],
                     bias_fmt=E5M2)


SPLIT_CASES = [
    # (layout, M, N, K, batch, bcast_b, bias_kind, fa, fb, split_k)
    (NT, 2048, 1024, 4096, 1, False, 0, E4M3, E4M3, 2),
    (NN, 2048, 1024, 3072, 1, False, 1, E5M2, E4M3, 2),   # a linear layer's dX shape, bf16 bias
    (TN, 1024, 1024, 2048, 1, False, 0, E5M2, E4M3, 4),   # a linear layer's dW shape
    (NT, 1000, 1008, 4096, 1, False, 2, E4M3, E4M3, 3),   # ragged M and N tails, fp8 bias
    (NT, 64, 8192, 2048, 1, False, 1, E4M3, E4M3, 4),     # skinny
    (NT, 1, 4096, 4096, 1, False, 0, E4M3, E5M2, 4),      # one row (decode)
    (NN, 8, 4096, 4096, 1, False, 0, E4M3, E4M3, 2),
    (NT, 256, 256, 4096, 3, True, 1, E4M3, E4M3, 3),      # batches with a broadcast B
    (TN, 384, 512, 2816, 2, False, 0, E5M2, E4M3, 3),     # ragged k split (22 k-blocks: 8, 8, 6)
]


@pytest.mark.parametrize("case", SPLIT_CASES, ids=lambda c: "x".join(map(str, c[:4])) + f"b{c[4]}s{c[9]}")
def test_split_matches_the_oracle(g, case):
    import fp8_delayed_scaling_quantize_b200 as fp8
    layout, M, N, K, batch, bcast_b, bias_kind, fa, fb, split_k = case
    need = fp8.fp8_mm_workspace_size(M, N, K, batch, layout, split_k)
    assert need > 4096
    c = _case(layout, M, N, K, fa, fb, 600 + M + K, batch, bcast_b, bias_kind)
    ws = g.workspace(need)
    out = _run(g, c, layout, M, N, K, fa, fb, batch, ws, split_k)
    y, s = _oracle(c, layout, M, N, K, fa, fb, batch)
    g.assert_within(out.float().cpu().numpy().reshape(y.shape), y, oracle.tolerance(y, s),
                    f"split {split_k} {layout} {M}x{N}x{K} b{batch}")
    assert not ws[:4096].any(), "counters must be zero after the call"
    # run to run: bit-identical
    again = _run(g, c, layout, M, N, K, fa, fb, batch, ws, split_k)
    assert torch.equal(out.view(torch.int16), again.view(torch.int16))
    assert fp8.fp8_last_device_error() == fp8.FP8_OK


def test_workspace_checks_and_no_split_is_fp8_mm(g):
    import fp8_delayed_scaling_quantize_b200 as fp8
    layout, M, N, K = NT, 2048, 1024, 4096
    c = _case(layout, M, N, K, E4M3, E4M3, 71)
    need = fp8.fp8_mm_workspace_size(M, N, K, 1, layout, 2)
    with pytest.raises(fp8.Fp8Error) as e:
        _run(g, c, layout, M, N, K, E4M3, E4M3, 1, g.workspace(need - 16), 2)
    assert e.value.status == fp8.FP8_ERR_INVALID_ARG
    with pytest.raises(fp8.Fp8Error) as e:
        _run(g, c, layout, M, N, K, E4M3, E4M3, 1, None, 2)
    assert e.value.status == fp8.FP8_ERR_INVALID_ARG
    # 16 k-blocks cannot be split 4 ways when K is 256
    with pytest.raises(fp8.Fp8Error) as e:
        _run(g, _case(layout, M, N, 256, E4M3, E4M3, 72), layout, M, N, 256, E4M3, E4M3, 1, g.workspace(1 << 26), 4)
    assert e.value.status == fp8.FP8_ERR_UNSUPPORTED
    plain = _run(g, c, layout, M, N, K, E4M3, E4M3, 1, None)
    for split_k in (0, 1):
        assert fp8.fp8_mm_workspace_size(M, N, K, 1, layout, split_k) == 0
        nows = _run(g, c, layout, M, N, K, E4M3, E4M3, 1, g.workspace(4096), split_k)
        assert torch.equal(plain.view(torch.int16), nows.view(torch.int16))


def test_one_workspace_serves_a_sequence_and_graph_replay(g):
    """The stack's split GEMMs one after another on one workspace, eager and
    then replayed from a CUDA graph: every output equals its first eager run
    bit for bit, and the counters end at zero."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    probs = [(NT, 2048, 1024, 4096), (NN, 2048, 1024, 4096), (NN, 2048, 1024, 3072), (TN, 1024, 1024, 2048)]
    need = max(fp8.fp8_mm_workspace_size(M, N, K, 1, l, 2) for l, M, N, K in probs)
    ws = g.workspace(need)
    sa = torch.tensor([0.5], device="cuda")
    sb = torch.tensor([2.0], device="cuda")
    ins, outs = [], []
    for i, (l, M, N, K) in enumerate(probs):
        a8 = W.fp8_codes((M * K,), E4M3, 900 + i).cuda()
        b8 = W.fp8_codes((N * K,), E4M3, 950 + i).cuda()
        ins.append((a8, b8))
        outs.append(torch.empty(M * N, dtype=torch.bfloat16, device="cuda"))

    def seq(stream=None):
        for (l, M, N, K), (a8, b8), o in zip(probs, ins, outs):
            fp8.fp8_mm_ws(a8, E4M3, b8, E4M3, sa, sb, l, M, N, K, 1, M * K, N * K, M * N, None, None, 0, o, ws,
                          2, stream=stream)

    seq()
    torch.cuda.synchronize()
    first = [o.clone() for o in outs]
    for (l, M, N, K), (a8, b8), o in zip(probs, ins, first):
        y, s = oracle.mm(a8.cpu().numpy(), E4M3, b8.cpu().numpy(), E4M3, 0.5, 2.0, l, M, N, K)
        g.assert_within(o.float().cpu().numpy().reshape(M, N), y, oracle.tolerance(y, s), f"{l} {M}x{N}x{K}")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            seq(stream)
    torch.cuda.synchronize()
    for _ in range(3):
        for o in outs:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for o, f in zip(outs, first):
            assert torch.equal(o.view(torch.int16), f.view(torch.int16))
        assert not ws[:4096].any()
    del graph
    assert fp8.fp8_last_device_error() == fp8.FP8_OK


@pytest.mark.parametrize("layout,M,N,K", [(NT, 1, 4096, 4096), (NN, 8, 4096, 4096), (NT, 16, 8192, 8192)])
def test_automatic_split_of_short_problems(g, layout, M, N, K):
    """split_k = 0 with a workspace: short problems with a long K split on
    their own (the workspace size query says how much they need); the result
    is the oracle's, bit-identical run to run, and fp8_mm (no workspace)
    gives the same bits."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    need = fp8.fp8_mm_workspace_size(M, N, K, 1, layout, 0)
    assert need > 4096, "the automatic choice is expected to split this shape"
    c = _case(layout, M, N, K, E4M3, E4M3, 1700 + M)
    ws = g.workspace(need)
    out = _run(g, c, layout, M, N, K, E4M3, E4M3, 1, ws, 0)
    again = _run(g, c, layout, M, N, K, E4M3, E4M3, 1, ws, 0)
    assert torch.equal(out.view(torch.int16), again.view(torch.int16))
    assert not ws[:4096].any()
    y, s = _oracle(c, layout, M, N, K, E4M3, E4M3, 1)
    tol = oracle.tolerance(y, s)
    g.assert_within(out.float().cpu().numpy().reshape(y.shape), y, tol, f"auto split {M}x{N}x{K}")
    # fp8_mm (no workspace) splits the same way as a cluster, the other splits'
    # partials reaching split 0 through its shared memory: the same sum in the
    # same order, so the same bits
    plain = _run(g, c, layout, M, N, K, E4M3, E4M3, 1, None, 0)
    assert torch.equal(plain.view(torch.int16), out.view(torch.int16))


# Cluster splits of short problems (fp8_mm, no workspace): ragged N, bias,
# batches with B broadcast; 16-row tiles split up to 4 ways, 32-row tiles 2
# ways. Against the oracle in full and the workspace split with the same
# number of splits bit for bit.
@pytest.mark.parametrize("layout,M,N,K,batch,bias_kind,split", [
    (NT, 5, 1000, 4096, 2, 1, 4), (NN, 12, 2048, 3072, 1, 2, 4), (NT, 24, 2048, 4096, 1, 1, 2),
    (NN, 32, 1024, 8192, 1, 0, 2)])
def test_cluster_split_of_short_problems(g, layout, M, N, K, batch, bias_kind, split):
    import fp8_delayed_scaling_quantize_b200 as fp8
    c = _case(layout, M, N, K, E4M3, E5M2, 1800 + M + N, batch=batch, bcast_b=batch > 1, bias_kind=bias_kind)
    plain = _run(g, c, layout, M, N, K, E4M3, E5M2, batch, None, 0)
    ws = g.workspace(fp8.fp8_mm_workspace_size(M, N, K, batch, layout, split))
    forced = _run(g, c, layout, M, N, K, E4M3, E5M2, batch, ws, split)
    assert torch.equal(plain.view(torch.int16), forced.view(torch.int16))
    y, s = _oracle(c, layout, M, N, K, E4M3, E5M2, batch)
    g.assert_within(plain.float().cpu().numpy().reshape(y.shape), y, oracle.tolerance(y, s),
                    f"cluster split {M}x{N}x{K}")
    assert fp8.fp8_last_device_error() == fp8.FP8_OK


def test_cluster_split_in_a_cuda_graph(g):
    """A short problem that splits as a cluster, captured in a CUDA graph and
    replayed on new operands: every replay equals a fresh eager call."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    M, N, K = 8, 2048, 4096
    c = _case(NT, M, N, K, E4M3, E4M3, 1900)
    a, b = c["a8"].cuda(), c["b8"].cuda()
    sa = torch.tensor([0.75], device="cuda")
    sb = torch.tensor([1.5], device="cuda")
    out = torch.empty(M * N, dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        g.mm(a, E4M3, b, E4M3, sa, sb, NT, M, N, K, out=out)
    torch.cuda.current_stream().wait_stream(st)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        g.mm(a, E4M3, b, E4M3, sa, sb, NT, M, N, K, out=out)
    for seed in (1901, 1902, 1903):
        a.copy_(W.fp8_codes((M * K,), E4M3, seed).cuda())
        graph.replay()
        want = _run(g, dict(c, a8=a.cpu()), NT, M, N, K, E4M3, E4M3, 1, None, 0)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), want.view(torch.int16))
    del graph
    assert fp8.fp8_last_device_error() == fp8.FP8_OK
