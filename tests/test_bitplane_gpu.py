"""GPU parity of the ternary-weight x 1-bit-activation bit-plane GEMV (and
its planes) against the CPU oracle, through the C ABI: planes and int32
accumulators bit for bit, outputs within 1e-3 relative and bit-identical."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from parity_helpers import compare_outputs, dev, oracle_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_ternary_weight_b200 as b
    return b


@pytest.mark.parametrize("N,K", [(28672, 8192), (8192, 28672), (6912, 2560), (333, 640),
                                 (1, 64), (10, 65536), (1001, 192)])
@pytest.mark.parametrize("xdtype,out_dtype", [(torch.bfloat16, torch.bfloat16),
                                              (torch.float32, torch.float32)])
def test_bitplane_gemv_parity(bl, N, K, xdtype, out_dtype):
    W = si.weight(N, K, seed=N + 3 * K)
    g, codes, _ = oracle_weight(W)
    x = si.activations(1, K, seed=K, dtype=xdtype)
    ref = oracle.bitplane_gemv(codes, g, x.float().numpy())
    w = bl.pack(W.to(dev()))
    bp = bl.bitplane_pack(w)
    acc = torch.empty(N, dtype=torch.int32, device=dev())
    y = bl.bitplane_gemv(bp, x.to(dev()), out_dtype=out_dtype, acc_dbg=acc)
    torch.cuda.synchronize()
    planes = bp.planes.cpu().numpy().view(np.uint64)
    np.testing.assert_array_equal(planes[:, :, 0], ref["mag"])
    np.testing.assert_array_equal(planes[:, :, 1], ref["sign"])
    np.testing.assert_array_equal(acc.cpu().numpy(), ref["acc"])
    compare_outputs(y.view(1, N), ref["y"].reshape(1, N))
    assert bl.last_device_status() == 0


def test_bitplane_zero_and_signed_zero_activations(bl):
    N, K = 200, 1024
    W = si.weight(N, K, seed=5)
    g, codes, _ = oracle_weight(W)
    x = si.activations(1, K, seed=6, dtype=torch.float32)
    x[0, ::7] = 0.0
    x[0, 3::11] = -0.0
    ref = oracle.bitplane_gemv(codes, g, x.numpy())
    bp = bl.bitplane_pack(bl.pack(W.to(dev())))
    acc = torch.empty(N, dtype=torch.int32, device=dev())
    y = bl.bitplane_gemv(bp, x.to(dev()), acc_dbg=acc)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(acc.cpu().numpy(), ref["acc"])
    compare_outputs(y.view(1, N), ref["y"].reshape(1, N))
