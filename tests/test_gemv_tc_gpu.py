"""Small-batch ternary GEMV on the tensor cores (2 .. 16 tokens, gemv_tc.cu)
against the oracle, next to the dp4a multi-token kernel on the same inputs.

The shapes reach every cluster split the launcher picks (one CTA per row
block up to eight CTAs sharing a block's k range), ragged row counts (a
partial last 128-row block and a partial last 8-row group), several products
in one launch, and pre-quantised activations; the integer accumulators must
equal the oracle's exactly and the outputs be the oracle's bf16 values.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from parity_helpers import compare_outputs, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import bit_ternary_weight_b200 as m
    return m


def _oracle(W, x):
    W = W.float().numpy()
    g = oracle.weight_scale(W)
    codes = oracle.ternary_codes(W, g)
    q, d, r = oracle.quantize_act(x.float().numpy())
    acc = oracle.ternary_acc(codes, q)
    return acc, oracle.rescale(acc, d, g)


def _run(bl, Ns, K, M, seed, dp4a, xdtype=torch.bfloat16):
    x = si.activations(M, K, seed=seed, dtype=xdtype)
    Ws = [si.weight(N, K, seed=seed + 11 * i + N) for i, N in enumerate(Ns)]
    ws = [bl.pack(W.to(dev())) for W in Ws]
    accs = [torch.empty(M, N, dtype=torch.int32, device=dev()) for N in Ns]
    big = [torch.full((M, N + 24), -5.0, dtype=torch.bfloat16, device=dev()) for N in Ns]
    outs = [b[:, :N] for b, N in zip(big, Ns)]
    bl.gemv_fused_multi(ws, x.to(dev()), outs=outs, acc_dbgs=accs, small_batch="dp4a" if dp4a else "tensor")
    torch.cuda.synchronize()
    for W, y, acc, b, N in zip(Ws, outs, accs, big, Ns):
        acc_o, y_o = _oracle(W, x)
        np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
        compare_outputs(y, y_o)
        assert (b[:, N:] == -5.0).all(), "written past the row"
    assert bl.last_device_status() == 0


@pytest.mark.parametrize("M", [2, 3, 4, 7, 8, 9, 15, 16])
@pytest.mark.parametrize("K,Ns", [(2560, [6912]), (6912, [2560]), (2560, [2560]), (2560, [640]),
                                  (2560, [2560, 640, 640])])
def test_tensor_core_small_batch_2b_shapes(bl, M, K, Ns):
    """The 2.4B layer shapes: the tensor-core kernel (default) and the dp4a
    multi-token kernel (flag) both equal the oracle."""
    assert bl.gemv_plan(Ns, K, M, small_batch="tensor")[0] == "tensor"
    assert bl.gemv_plan(Ns, K, M, small_batch="dp4a")[0] == "stream_mt"
    assert bl.gemv_plan(Ns, K, M)[0] in ("tensor", "stream_mt")
    _run(bl, Ns, K, M, seed=900 + M + K, dp4a=False)
    _run(bl, Ns, K, M, seed=900 + M + K, dp4a=True)


@pytest.mark.parametrize("K,Ns,cs", [
    (256, [1001], 1),          # one stage: one CTA per block
    (512, [300], 2),           # two stages, one per CTA of a pair
    (1024, [129], 4),          # a block of one row past 128
    (2048, [8, 1000], 8),      # two products, one of a single group; one stage per CTA
    (7936, [1000], 8),         # 31 stages: eight CTAs per block, three or four stages each
    (1536, [12800], None),     # six stages, 100 blocks: the split the device's capacity allows
])
@pytest.mark.parametrize("M", [2, 16])
def test_tensor_core_cluster_splits_and_ragged_rows(bl, K, Ns, cs, M):
    kern, got = bl.gemv_plan(Ns, K, M, small_batch="tensor")
    assert kern == "tensor"
    if cs is not None:
        assert got == cs
    _run(bl, Ns, K, M, seed=77 + K + M, dp4a=False)


def test_tensor_core_prequantised(bl):
    """bitlinear_gemv (pre-quantised q, d, rowsum) takes the tensor-core kernel
    past the crossover too; partial row sums come from q itself."""
    for M, K, N in [(4, 2560, 6912), (5, 6912, 2560), (16, 1024, 4001)]:
        assert bl.gemv_plan([N], K, M, fused=False)[0] == "tensor"
        x = si.activations(M, K, seed=M + K)
        W = si.weight(N, K, seed=N + M)
        w = bl.pack(W.to(dev()))
        q, d, r = bl.quantize_act(x.to(dev()))
        acc = torch.empty(M, N, dtype=torch.int32, device=dev())
        y = bl.gemv(w, q, d, r, acc_dbg=acc)
        torch.cuda.synchronize()
        acc_o, y_o = _oracle(W, x)
        np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
        compare_outputs(y, y_o)
    assert bl.last_device_status() == 0


def test_tensor_core_edge_tokens(bl):
    """A zero token, a token of one huge outlier and a tiny token in one batch."""
    K, N, M = 2560, 2560, 4
    x = si.activations(M, K, seed=5)
    x[0] = 0
    x[1] = 0
    x[1, 1234] = 3.0e4
    x[2] = x[2] * 1e-30
    W = si.weight(N, K, seed=6)
    w = bl.pack(W.to(dev()))
    acc = torch.empty(M, N, dtype=torch.int32, device=dev())
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev())
    bl.gemv_fused_multi([w], x.to(dev()), outs=[y], acc_dbgs=[acc], small_batch="tensor")
    torch.cuda.synchronize()
    acc_o, y_o = _oracle(W, x)
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    compare_outputs(y, y_o)


def test_tensor_core_chain_in_graph_with_pdl(bl):
    """Sixteen tokens through a four-deep dependent chain of tensor-core
    launches with programmatic dependent launch, captured in a CUDA graph:
    every link equals the oracle applied to the previous link's output."""
    K, M = 2560, 16
    Ws = [si.weight(K, K, seed=300 + i) for i in range(4)]
    ws = [bl.pack(W.to(dev())) for W in Ws]
    x0 = si.activations(M, K, seed=301)
    xs = [x0.to(dev())] + [torch.empty(M, K, dtype=torch.bfloat16, device=dev()) for _ in Ws]

    def run():
        for i, w in enumerate(ws):
            bl.gemv_fused_multi([w], xs[i], outs=[xs[i + 1]], pdl=True, small_batch="tensor")
    run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for t in xs[1:]:
        t.fill_(0)
    g.replay()
    torch.cuda.synchronize()
    for i, W in enumerate(Ws):
        _, y_o = _oracle(W, xs[i].cpu())
        compare_outputs(xs[i + 1], y_o)
    del g
    assert bl.last_device_status() == 0


def test_default_routing_follows_the_crossover(bl):
    """The default picks the tensor cores past M N K = 48 Mi or K > 4096."""
    assert bl.gemv_plan([6912], 2560, 2)[0] == "stream_mt"      # 35 Mi
    assert bl.gemv_plan([6912], 2560, 4)[0] == "tensor"         # 71 Mi
    assert bl.gemv_plan([2560], 6912, 2)[0] == "tensor"         # K > 4096
    assert bl.gemv_plan([640], 2560, 16)[0] == "stream_mt"      # 26 Mi
    assert bl.gemv_plan([6912], 2560, 1)[0] == "stream"
