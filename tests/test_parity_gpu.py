"""GPU parity of the CUDA path against the CPU oracle, through the C ABI.

Integers (packed bytes, q, rowsum, acc) must match bit for bit; the weight
and activation scales must match bit for bit (they are defined with a fixed
fp32/fp64 operation order); rescaled outputs must be within 1e-3 relative of
the oracle and, by construction, bit-identical to it.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from parity_helpers import (Guarded, compare_outputs, dev, f32_bits, oracle_weight,
                            seeded_problem)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_ternary_weight_b200 as b
    return b


def _pack_gpu(bl, W):
    return bl.pack(W.to(dev()))


# ------------------------------------------------------------------ packer

PACK_SHAPES = [(8, 64), (13, 128), (40, 2560), (512, 256), (1001, 192),
               (2560, 2560), (640, 2560), (6912, 2560), (2560, 6912)]


@pytest.mark.parametrize("N,K", PACK_SHAPES)
@pytest.mark.parametrize("wdtype", [torch.float32, torch.bfloat16])
def test_pack_parity(bl, N, K, wdtype):
    W = si.weight(N, K, seed=N + K).to(wdtype)
    g, codes, packed = oracle_weight(W.float())
    w = _pack_gpu(bl, W)
    torch.cuda.synchronize()
    assert f32_bits(w.w_scale.cpu().numpy())[0] == f32_bits(np.float32([g]))[0]
    np.testing.assert_array_equal(w.packed.cpu().numpy(), packed)


@pytest.mark.parametrize("N,K", [(28672, 8192), (8192, 28672)])
def test_pack_parity_100b(bl, N, K):
    W = si.weight(N, K, seed=7)
    g, codes, packed = oracle_weight(W)
    w = _pack_gpu(bl, W)
    torch.cuda.synchronize()
    assert f32_bits(w.w_scale.cpu().numpy())[0] == f32_bits(np.float32([g]))[0]
    np.testing.assert_array_equal(w.packed.cpu().numpy(), packed)


def test_pack_zero_weight(bl):
    W = torch.zeros(16, 128)
    w = _pack_gpu(bl, W)
    assert w.w_scale.item() == np.float32(1e-5)
    assert (w.packed.cpu().numpy() == 0x55).all()


# ------------------------------------------------------------------ activation quant

@pytest.mark.parametrize("M,K", [(1, 256), (3, 2560), (16, 6912), (128, 256), (512, 2560),
                                 (2, 28672), (8192, 6912), (8192, 2560), (1024, 2048), (1031, 3072),
                                 (2048, 320)])
@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float32])
def test_quantize_parity(bl, M, K, xdtype):
    x = si.activations(M, K, seed=M + K, dtype=xdtype)
    q_o, d_o, r_o = oracle.quantize_act(x.float().numpy())
    q, d, r = bl.quantize_act(x.to(dev()))
    np.testing.assert_array_equal(q.cpu().numpy(), q_o)
    np.testing.assert_array_equal(f32_bits(d.cpu().numpy()), f32_bits(d_o))
    np.testing.assert_array_equal(r.cpu().numpy(), r_o)


def test_quantize_edge_tokens(bl):
    K = 512
    x = torch.randn(6, K)
    x[0] = 0.0                       # all-zero token
    x[1, 17] = 1e4                   # one huge outlier
    x[2] = 3.0                       # constant token: every q = 127
    x[2, ::2] = -3.0
    x[3] = 1e-30                     # below the 1e-5 floor
    x[4] = torch.tensor([2.5, -1.5] * (K // 2))  # exact halves after scaling
    x[4, 0] = 127.0
    x[5, 5] = -x[5].abs().max() * 2  # negative extreme
    for xd in (torch.float32, torch.bfloat16):
        xx = x.to(xd)
        q_o, d_o, r_o = oracle.quantize_act(xx.float().numpy())
        q, d, r = bl.quantize_act(xx.to(dev()))
        np.testing.assert_array_equal(q.cpu().numpy(), q_o)
        np.testing.assert_array_equal(f32_bits(d.cpu().numpy()), f32_bits(d_o))
        np.testing.assert_array_equal(r.cpu().numpy(), r_o)


def test_quantize_many_short_rows_edge_tokens(bl):
    """The warp-per-token kernel (bf16, many rows, K <= 3072) on the edge
    tokens of test_quantize_edge_tokens, spread over 1500 rows of a strided
    view, with a ragged K (a last lane chunk only partly used)."""
    M, K, ld = 1500, 2368, 2560
    base = si.activations(M, ld, seed=11, dtype=torch.bfloat16)
    x = base[:, :K].clone()
    x[0] = 0.0
    x[77, 17] = 1e4
    x[500] = 3.0
    x[500, ::2] = -3.0
    x[1001] = 1e-30
    x[1499, 5] = -x[1499].abs().max() * 2
    base[:, :K] = x
    q_o, d_o, r_o = oracle.quantize_act(x.float().numpy())
    q, d, r = bl.quantize_act(base.to(dev())[:, :K])
    np.testing.assert_array_equal(q.cpu().numpy(), q_o)
    np.testing.assert_array_equal(f32_bits(d.cpu().numpy()), f32_bits(d_o))
    np.testing.assert_array_equal(r.cpu().numpy(), r_o)


def test_quantize_strided_rows(bl):
    M, K, ld = 5, 256, 384
    base = si.activations(M, ld, seed=3, dtype=torch.bfloat16)
    x = base[:, :K]
    q_o, d_o, r_o = oracle.quantize_act(x.float().numpy())
    q, d, r = bl.quantize_act(base.to(dev())[:, :K])
    np.testing.assert_array_equal(q.cpu().numpy(), q_o)
    np.testing.assert_array_equal(r.cpu().numpy(), r_o)


# ------------------------------------------------------------------ ternary GEMV

def _oracle_gemv(g, codes, x):
    q, d, r = oracle.quantize_act(x.float().numpy())
    acc = oracle.ternary_acc(codes, q)
    return oracle.rescale(acc, d, g), acc


def _check_gemv(bl, W, x, out_dtype, fused, guard=True):
    N, K = W.shape
    M = x.shape[0]
    g, codes, _ = oracle_weight(W)
    y_o, acc_o = _oracle_gemv(g, codes, x)
    w = _pack_gpu(bl, W)
    xd = x.to(dev())
    yb = Guarded(M * N, out_dtype, dev())
    ab = Guarded(M * N, torch.int32, dev())
    y = yb.view.view(M, N)
    acc = ab.view.view(M, N)
    if fused:
        bl.gemv_fused(w, xd, out=y, acc_dbg=acc)
    else:
        q, d, r = bl.quantize_act(xd)
        bl.gemv(w, q, d, r, out=y, acc_dbg=acc)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    compare_outputs(y, y_o)
    if guard:
        assert yb.intact() and ab.intact()


@pytest.mark.parametrize("K,N", si.DECODE_SHAPES_2B)
@pytest.mark.parametrize("fused", [True, False])
def test_decode_gemv_2b_shapes(bl, K, N, fused):
    W, x = seeded_problem(N, K, 1, seed=0)
    _check_gemv(bl, W, x, torch.bfloat16, fused)


@pytest.mark.parametrize("K,N", si.DECODE_SHAPES_2B)
def test_decode_gemv_fp32_output(bl, K, N):
    W, x = seeded_problem(N, K, 1, seed=1)
    _check_gemv(bl, W, x, torch.float32, True)


@pytest.mark.parametrize("K,N", si.DECODE_SHAPES_100B)
def test_decode_gemv_100b_shapes(bl, K, N):
    W, x = seeded_problem(N, K, 1, seed=0)
    _check_gemv(bl, W, x, torch.bfloat16, True)


# One token on a large layer (K a multiple of 4096, at least four row groups
# per SM) runs the producer/consumer streaming kernel: both 100B shapes,
# fp32 and bf16 activations, pre-quantised q, fp32 output, ragged N whose
# last set of groups is short, K = 32768 (the largest register-resident
# quantisation) and 64 row groups per CTA (its shared row-sum capacity).
@pytest.mark.parametrize("N,K,fused,xdtype,out_dtype", [
    (28672, 8192, True, torch.bfloat16, torch.bfloat16),
    (8192, 28672, True, torch.float32, torch.bfloat16),
    (8192, 28672, False, torch.bfloat16, torch.float32),
    (4739, 4096, False, torch.bfloat16, torch.bfloat16),
    (4739, 32768, True, torch.bfloat16, torch.bfloat16),
    (4745, 8192, True, torch.float32, torch.float32),
    (75776, 4096, True, torch.bfloat16, torch.bfloat16),
])
def test_gemv_stream_kernel(bl, N, K, fused, xdtype, out_dtype):
    W, x = seeded_problem(N, K, 1, seed=N + K, xdtype=xdtype)
    _check_gemv(bl, W, x, out_dtype, fused)


# One token with K a multiple of 256 always runs the streaming kernel: ragged
# last stages (K = 2304: 9 pieces of 256 k; 768: 3; 256: 1), products of
# mixed sizes whose concatenated row groups straddle product boundaries inside
# a CTA's sets, eight products at once, small and large launches.
@pytest.mark.parametrize("Ns,K,fused,xdtype", [
    ([1001], 2304, True, torch.bfloat16),
    ([8], 256, False, torch.bfloat16),
    ([1], 768, True, torch.float32),
    ([4739], 2304, False, torch.bfloat16),
    ([2000, 3001, 17, 4500], 1280, True, torch.bfloat16),
    ([640, 13, 2560, 999, 64, 7, 1500, 3], 6912, True, torch.float32),
    ([6912, 6912], 2560, True, torch.bfloat16),
])
def test_gemv_stream_products_and_ragged_k(bl, Ns, K, fused, xdtype):
    x = si.activations(1, K, seed=K + len(Ns), dtype=xdtype)
    ws, refs = [], []
    for i, N in enumerate(Ns):
        W = si.weight(N, K, seed=900 + 7 * i + N)
        g, codes, _ = oracle_weight(W)
        refs.append(_oracle_gemv(g, codes, x))
        ws.append(_pack_gpu(bl, W))
    accs = [torch.empty(1, N, dtype=torch.int32, device=dev()) for N in Ns]
    xd = x.to(dev())
    if fused:
        outs = bl.gemv_fused_multi(ws, xd, acc_dbgs=accs)
    else:
        assert len(ws) == 1
        q, d, r = bl.quantize_act(xd)
        outs = [bl.gemv(ws[0], q, d, r, acc_dbg=accs[0])]
    torch.cuda.synchronize()
    for (y_o, acc_o), y, acc in zip(refs, outs, accs):
        np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
        compare_outputs(y, y_o)
    assert bl.last_device_status() == 0


@pytest.mark.parametrize("N,K,M", [(13, 64, 1), (1001, 192, 3), (8, 128, 16), (77, 320, 5),
                                   (1, 64, 2), (4096, 64, 7), (24, 10240, 16)])
@pytest.mark.parametrize("fused", [True, False])
def test_gemv_ragged_and_edge(bl, N, K, M, fused):
    W, x = seeded_problem(N, K, M, seed=N * 7 + K + M)
    if M >= 2:
        x[0] = 0.0
    _check_gemv(bl, W, x, torch.bfloat16, fused)


@pytest.mark.parametrize("M", [8, 16])
def test_small_batch_tensor_core_path(bl, M):
    """bitlinear_gemv and linear() at 8 and 16 tokens (the tcgen05 path for
    16 tokens on weights above 4M entries, the multi-token streaming kernel
    otherwise): the four 2.4B shapes x 10 seeds, integers bit-exact, outputs
    equal."""
    for K, N in si.DECODE_SHAPES_2B:
        for seed in range(10):
            W = si.weight(N, K, seed=2000 + seed)
            g, codes, _ = oracle_weight(W)
            w = _pack_gpu(bl, W)
            x = si.activations(M, K, seed=seed * 17 + M)
            y_o, acc_o = _oracle_gemv(g, codes, x)
            xd = x.to(dev())
            q, d, r = bl.quantize_act(xd)
            acc = torch.empty(M, N, dtype=torch.int32, device=dev())
            y = bl.gemv(w, q, d, r, acc_dbg=acc)
            np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
            compare_outputs(y, y_o)
            compare_outputs(bl.linear(w, xd), y_o)


def test_gemv_fp32_input_and_strided_output(bl):
    N, K, M = 300, 256, 4
    W, x = seeded_problem(N, K, M, seed=11, xdtype=torch.float32)
    g, codes, _ = oracle_weight(W)
    y_o, _ = _oracle_gemv(g, codes, x)
    w = _pack_gpu(bl, W)
    big = torch.full((M, 320), -7.0, dtype=torch.float32, device=dev())
    bl.gemv_fused(w, x.to(dev()), out=big[:, :N])
    torch.cuda.synchronize()
    compare_outputs(big[:, :N], y_o)
    assert (big[:, N:] == -7.0).all()


def test_small_batch_sweep_100_seeds(bl):
    """Small-batch GEMV: M in {1,2,4,8,16} x the four 2.4B shapes x 100 seeds."""
    for K, N in si.DECODE_SHAPES_2B:
        for seed in range(100):
            W = si.weight(N, K, seed=1000 + seed)
            g, codes, _ = oracle_weight(W)
            w = _pack_gpu(bl, W)
            for M in si.SMALL_BATCH_M:
                x = si.activations(M, K, seed=seed * 31 + M)
                y_o, acc_o = _oracle_gemv(g, codes, x)
                acc = torch.empty(M, N, dtype=torch.int32, device=dev())
                y = bl.gemv_fused(w, x.to(dev()), acc_dbg=acc)
                np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
                compare_outputs(y, y_o)


def test_host_pointer_rejected(bl):
    W = si.weight(16, 64)
    w = _pack_gpu(bl, W)
    x_host = torch.randn(1, 64, dtype=torch.bfloat16)
    with pytest.raises(bl.BitLinearError) as e:
        bl.gemv_fused(w, x_host, out=torch.empty(1, 16, dtype=torch.bfloat16, device=dev()))
    assert e.value.status == bl.BL_ERR_NOT_DEVICE_PTR


# ------------------------------------------------------------------ binary GEMV

@pytest.mark.parametrize("N,K", [(28672, 8192), (1, 64), (333, 640), (64, 4096), (10, 40960)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_binary_gemv_parity(bl, N, K, out_dtype):
    W = si.weight(N, K, seed=K)
    x = si.activations(1, K, seed=K, dtype=torch.bfloat16)
    ref = oracle.binary_gemv(W.numpy(), x.float().numpy())
    bw = bl.binary_pack(W.to(dev()))
    acc = torch.empty(N, dtype=torch.int32, device=dev())
    y = bl.binary_gemv(bw, x.to(dev()), out_dtype=out_dtype, acc_dbg=acc)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bw.bits.cpu().numpy().view(np.uint64), ref["Wb"])
    assert f32_bits(bw.s_w.cpu().numpy())[0] == f32_bits(np.float32([ref["s_w"]]))[0]
    np.testing.assert_array_equal(acc.cpu().numpy(), ref["acc"])
    compare_outputs(y.view(1, N), ref["y"].reshape(1, N))


# ------------------------------------------------------------------ prefill GEMM (tcgen05)

def _check_gemm(bl, N, K, M, xdtype=torch.bfloat16, out_dtype=torch.bfloat16, seed=0,
                outliers=True, sample=None):
    W = si.weight(N, K, seed=seed)
    x = si.activations(M, K, seed=seed, outliers=outliers, dtype=xdtype)
    g, codes, _ = oracle_weight(W)
    w = _pack_gpu(bl, W)
    q, d, r = bl.quantize_act(x.to(dev()))
    yb = Guarded(M * N, out_dtype, dev())
    ab = Guarded(M * N, torch.int32, dev())
    y = yb.view.view(M, N)
    acc = ab.view.view(M, N)
    bl.gemm(w, q, d, r, out=y, acc_dbg=acc)
    torch.cuda.synchronize()
    assert bl.last_device_status() == 0
    rows = np.arange(M) if sample is None else sample
    xs = x[torch.as_tensor(rows)].float().numpy()
    q_o, d_o, r_o = oracle.quantize_act(xs)
    acc_o = oracle.ternary_acc(codes, q_o)
    y_o = oracle.rescale(acc_o, d_o, g)
    np.testing.assert_array_equal(acc.cpu().numpy()[rows], acc_o)
    compare_outputs(y[torch.as_tensor(rows, device=dev())], y_o)
    assert yb.intact() and ab.intact()


def test_gemm_config1_fp32(bl):
    """X[128x256] fp32 ~N(0,1) (no outliers) x W[512x256]^T, fp32 output."""
    _check_gemm(bl, 512, 256, 128, xdtype=torch.float32, out_dtype=torch.float32, outliers=False)


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (160, 200, 2560), (130, 300, 192),
                                   (256, 256, 64), (128, 1001, 320), (5, 77, 128),
                                   (300, 129, 6912), (17, 8, 64)])
def test_gemm_ragged_shapes(bl, M, N, K):
    _check_gemm(bl, N, K, M, seed=M + N + K)


@pytest.mark.parametrize("M,N,K", [(1200, 4000, 320), (1024, 2560, 1024), (2048, 2048, 128),
                                   (1100, 2900, 192)])
def test_gemm_several_tiles_per_cta(bl, M, N, K):
    """More output tiles than SMs: each persistent CTA walks several tiles,
    alternating its two accumulator buffers; every output is checked."""
    _check_gemm(bl, N, K, M, seed=M ^ N ^ K)


@pytest.mark.parametrize("M,N,K", [(1, 6912, 2560), (8, 6912, 2560), (16, 2560, 6912),
                                   (32, 2560, 6912), (3, 300, 320), (17, 1000, 1280)])
def test_gemm_split_k_small_batches(bl, M, N, K):
    """Small batches split K across CTAs and meet in the int32 workspace:
    bit-exact, the workspace is left zero, and a second call reusing it is
    exact too."""
    need = bl.gemm_workspace_bytes(M, N, K)
    assert need > 0
    W = si.weight(N, K, seed=M * 13 + N)
    x = si.activations(M, K, seed=M + K)
    g, codes, _ = oracle_weight(W)
    w = _pack_gpu(bl, W)
    q, d, r = bl.quantize_act(x.to(dev()))
    q_o, d_o, r_o = oracle.quantize_act(x.float().numpy())
    acc_o = oracle.ternary_acc(codes, q_o)
    y_o = oracle.rescale(acc_o, d_o, g)
    ws = torch.zeros(need, dtype=torch.uint8, device=dev())
    for _ in range(2):
        acc = torch.full((M, N), 7, dtype=torch.int32, device=dev())
        y = bl.gemm(w, q, d, r, acc_dbg=acc, workspace=ws)
        torch.cuda.synchronize()
        assert bl.last_device_status() == 0
        np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
        compare_outputs(y, y_o)
        assert int(torch.count_nonzero(ws)) == 0


def _tile_sample(M: int, seed: int, per_tile: int = 2) -> np.ndarray:
    """Token rows to check at full size: both edges of every 128-token tile
    boundary plus `per_tile` random tokens inside every tile, so that every
    (weight-row tile, token tile) pair of the persistent walk -- each CTA's
    first and last tile, and both accumulator buffers -- has checked outputs."""
    rng = np.random.default_rng(seed)
    rows = [0, M - 1]
    for t0 in range(0, M, 128):
        t1 = min(M, t0 + 128)
        rows += [t0, t1 - 1]
        rows += list(rng.integers(t0, t1, per_tile))
    return np.unique(np.asarray(rows, dtype=np.int64))


@pytest.mark.parametrize("K,N", si.PREFILL_SHAPES)
@pytest.mark.parametrize("M", si.PREFILL_TOKENS)
def test_gemm_prefill_full_size(bl, K, N, M):
    """Every output column of tokens drawn from every 128-token tile."""
    _check_gemm(bl, N, K, M, seed=3, sample=_tile_sample(M, M + K))


def test_gemm_prefill_every_output_m2048(bl):
    """Prefill 2048 tokens x (2560 -> 6912): every one of the 14.2 M outputs
    and int32 accumulators against the oracle (several tiles per CTA, both
    accumulator buffers, every ring wrap)."""
    _check_gemm(bl, 6912, 2560, 2048, seed=5)


def test_other_gpus_memory_rejected(bl):
    """A tensor on another GPU while cuda:0 is current: rejected before any
    launch (the raw C ABI, which does not switch devices)."""
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two GPUs")
    import ctypes
    w = _pack_gpu(bl, si.weight(16, 64))
    x1 = torch.zeros(1, 64, dtype=torch.bfloat16, device="cuda:1")
    y0 = torch.empty(1, 16, dtype=torch.bfloat16, device=dev())
    with torch.cuda.device(0):
        st = bl.lib.bitlinear_gemv_fused(
            ctypes.c_void_p(w.packed.data_ptr()), ctypes.c_void_p(w.w_scale.data_ptr()), 16, 64,
            ctypes.c_void_p(x1.data_ptr()), bl.BL_BF16, 64, 1, ctypes.c_void_p(y0.data_ptr()),
            bl.BL_BF16, 16, None, None)
    assert st == bl.BL_ERR_NOT_DEVICE_PTR


# ------------------------------------------------------------------ shared-input multi GEMV, PDL chains

@pytest.mark.parametrize("M", [1, 3, 16])
def test_multi_gemv_qkv_shapes(bl, M):
    """q/k/v of one 2.4B layer in one launch, each output against the oracle."""
    K = si.HIDDEN_2B
    shapes = [si.HIDDEN_2B, si.KV_2B, si.KV_2B]
    x = si.activations(M, K, seed=40 + M)
    ws, refs = [], []
    for i, N in enumerate(shapes):
        W = si.weight(N, K, seed=50 + i)
        g, codes, _ = oracle_weight(W)
        refs.append(_oracle_gemv(g, codes, x))
        ws.append(_pack_gpu(bl, W))
    accs = [torch.empty(M, N, dtype=torch.int32, device=dev()) for N in shapes]
    outs = bl.gemv_fused_multi(ws, x.to(dev()), acc_dbgs=accs)
    torch.cuda.synchronize()
    for (y_o, acc_o), y, acc in zip(refs, outs, accs):
        np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
        compare_outputs(y, y_o)


@pytest.mark.parametrize("K,M", [(2560, 1), (2560, 3), (8192, 1)])
def test_pdl_dependent_chain(bl, K, M):
    """A chain where each launch reads the previous launch's output, all with
    BL_FLAG_PDL, inside a CUDA graph (so that consecutive launches really
    overlap): the result must equal the oracle chain.  One token at K = 2560
    runs small streaming launches, three tokens the multi-token streaming
    kernel, one token at K = 8192 large streaming launches (two CTAs per SM)."""
    Ws = [si.weight(K, K, seed=70 + i) for i in range(6)]
    oracles = [oracle_weight(W) for W in Ws]
    ws = [_pack_gpu(bl, W) for W in Ws]
    x0 = si.activations(M, K, seed=77)
    xs = [x0.to(dev())] + [torch.empty(M, K, dtype=torch.bfloat16, device=dev()) for _ in Ws]
    for _ in range(2):  # warm-up, eager
        for i, w in enumerate(ws):
            bl.gemv_fused_multi([w], xs[i], outs=[xs[i + 1]], pdl=True)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i, w in enumerate(ws):
            bl.gemv_fused_multi([w], xs[i], outs=[xs[i + 1]], pdl=True)
    for i in range(1, len(xs)):
        xs[i].zero_()
    g.replay()
    torch.cuda.synchronize()
    x = x0
    for i, (gam, codes, _) in enumerate(oracles):
        y_o, _ = _oracle_gemv(gam, codes, x)
        compare_outputs(xs[i + 1], y_o)
        x = torch.from_numpy(oracle.to_bf16_bits(y_o).view(np.int16)).view(torch.bfloat16)
    assert bl.last_device_status() == 0


# ------------------------------------------------------------------ N-split (column-parallel) shards

@pytest.mark.parametrize("world,M", [(2, 1), (3, 1), (4, 1), (3, 3)])
def test_row_split_shards_equal_unsplit(bl, world, M):
    """Each rank's shard (a view of whole 8-row groups of the packed weight,
    the whole tensor's gamma) run through the fused multi-product GEMV into
    its slot of a gather buffer: the slots, laid end to end, are the unsplit
    outputs bit for bit.  All ranks are emulated on this one GPU, one after
    another; no rank waits on another."""
    from bit_ternary_weight_b200.sharding import row_partition, shard_weight
    K = si.HIDDEN_2B
    Ns = [si.HIDDEN_2B, si.KV_2B, 1001]
    x = si.activations(M, K, seed=600 + world)
    xd = x.to(dev())
    ws, refs = [], []
    for i, N in enumerate(Ns):
        W = si.weight(N, K, seed=610 + i)
        g, codes, _ = oracle_weight(W)
        refs.append(_oracle_gemv(g, codes, x)[0])
        ws.append(_pack_gpu(bl, W))
    parts = [row_partition(N, world) for N in Ns]
    bufs = [torch.full((world * M * p[0].rows_per_rank,), float("nan"), dtype=torch.bfloat16,
                       device=dev()) for p in parts]
    for r in range(world):
        live = []
        for w, p, buf in zip(ws, parts, bufs):
            sh = p[r]
            sw = shard_weight(w, sh)
            if sw is None:
                continue
            slot = buf[r * M * sh.rows_per_rank:(r + 1) * M * sh.rows_per_rank]
            live.append((sw, slot.view(M, sh.rows_per_rank)[:, :sh.rows]))
        if live:
            bl.gemv_fused_multi([a for a, _ in live], xd, outs=[b for _, b in live])
    torch.cuda.synchronize()
    for N, p, buf, y_o in zip(Ns, parts, bufs, refs):
        R = p[0].rows_per_rank
        full = buf.view(world, M, R).permute(1, 0, 2).reshape(M, world * R)[:, :N]
        compare_outputs(full, y_o)


# ------------------------------------------------------------------ small batches on the streaming kernel

@pytest.mark.parametrize("M", [2, 3, 5, 8, 13, 16])
@pytest.mark.parametrize("K,Ns", [(2560, [6912]), (6912, [2560]), (2560, [2560, 640, 640]),
                                  (256, [1001]), (8192, [3000])])
def test_small_batch_streaming_kernel(bl, M, K, Ns):
    """2 .. 16 tokens with K a multiple of 256 run the multi-token streaming
    kernel: fused (bf16 and fp32 x) for one or several products, and on
    pre-quantised activations (bitlinear_gemv, below 8 tokens), integers and
    outputs equal to the oracle's."""
    for xdtype in (torch.bfloat16, torch.float32):
        x = si.activations(M, K, seed=M * 31 + K, dtype=xdtype)
        ws, refs = [], []
        for i, N in enumerate(Ns):
            W = si.weight(N, K, seed=3000 + 17 * i + N + M)
            g, codes, _ = oracle_weight(W)
            refs.append(_oracle_gemv(g, codes, x))
            ws.append(_pack_gpu(bl, W))
        accs = [torch.empty(M, N, dtype=torch.int32, device=dev()) for N in Ns]
        big = [torch.full((M, N + 40), -3.0, dtype=torch.bfloat16, device=dev()) for N in Ns]
        outs = [b[:, :N] for b, N in zip(big, Ns)]
        bl.gemv_fused_multi(ws, x.to(dev()), outs=outs, acc_dbgs=accs)
        torch.cuda.synchronize()
        for (y_o, acc_o), y, acc, b, N in zip(refs, outs, accs, big, Ns):
            np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
            compare_outputs(y, y_o)
            assert (b[:, N:] == -3.0).all()
        if M < 8 and len(Ns) == 1:
            q, d, r = bl.quantize_act(x.to(dev()))
            acc = torch.empty(M, Ns[0], dtype=torch.int32, device=dev())
            y = bl.gemv(ws[0], q, d, r, acc_dbg=acc)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(acc.cpu().numpy(), refs[0][1])
            compare_outputs(y, refs[0][0])
    assert bl.last_device_status() == 0


def test_small_batch_pdl_chain_in_graph(bl):
    """Eight tokens through a six-deep dependent chain of launches (the
    tensor-core small-batch GEMV at this size) with programmatic dependent
    launch inside a CUDA graph."""
    K, M = 2560, 8
    Ws = [si.weight(K, K, seed=170 + i) for i in range(6)]
    oracles = [oracle_weight(W) for W in Ws]
    ws = [_pack_gpu(bl, W) for W in Ws]
    x0 = si.activations(M, K, seed=171)
    xs = [x0.to(dev())] + [torch.empty(M, K, dtype=torch.bfloat16, device=dev()) for _ in Ws]

    def run():
        for i, w in enumerate(ws):
            bl.gemv_fused_multi([w], xs[i], outs=[xs[i + 1]], pdl=True)
    run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for t in xs[1:]:
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    x = x0
    for i, (gam, codes, _) in enumerate(oracles):
        y_o, _ = _oracle_gemv(gam, codes, x)
        compare_outputs(xs[i + 1], y_o)
        x = torch.from_numpy(oracle.to_bf16_bits(y_o).view(np.int16)).view(torch.bfloat16).reshape(M, K)


def test_mma_probe_rate_is_plausible(bl):
    """The int8 tensor-core probe runs on every SM and reports a rate within
    the physically possible range (1 to 20 thousand MAC per clock per SM)."""
    r = bl.probe_mma_i8(reps=2000, device=dev())
    assert r["ctas"] == bl.sm_count()
    assert 1000 < r["mac_per_clk_per_sm"] < 20000
    assert bl.last_device_status() == 0


def test_narrow_mma_issue_probe(bl):
    """The 128 x 32 x 32 probe runs from 1, 2 and 4 warps; more issuers never
    lower the per-SM rate, and every rate is physically possible."""
    rates = [bl.probe_mma_i8(reps=2000, device=dev(), n=32, issuers=w)["mac_per_clk_per_sm"] for w in (1, 2, 4)]
    assert all(500 < r < 20000 for r in rates)
    assert rates[2] >= 0.9 * rates[0]
    assert bl.last_device_status() == 0
