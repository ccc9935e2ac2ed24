"""GPU parity of the lookup-table ternary GEMV against the CPU oracle (and
against the dp4a GEMV on the same inputs): int32 accumulators bit for bit,
outputs within 1e-3 relative and bit-identical."""
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


@pytest.mark.parametrize("N,K", [(N, K) for (K, N) in si.DECODE_SHAPES_2B]
                         + [(28672, 8192), (1001, 192), (1, 64), (77, 12288), (13, 320)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_lut_gemv_parity(bl, N, K, out_dtype):
    W = si.weight(N, K, seed=N ^ K)
    x = si.activations(1, K, seed=K + 1)
    g, codes, _ = oracle_weight(W)
    q_o, d_o, _ = oracle.quantize_act(x.float().numpy())
    acc_o = oracle.ternary_acc(codes, q_o)
    y_o = oracle.rescale(acc_o, d_o, g)
    w = bl.pack(W.to(dev()))
    q, d, r = bl.quantize_act(x.to(dev()))
    acc = torch.empty(1, N, dtype=torch.int32, device=dev())
    y = bl.lut_gemv(w, q, d, out_dtype=out_dtype, acc_dbg=acc)
    y_dp4a = bl.gemv(w, q, d, r, out_dtype=out_dtype)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    compare_outputs(y, y_o)
    assert torch.equal(y.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32),
                       y_dp4a.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32))


def test_lut_gemv_extreme_activations(bl):
    """q = +-127 everywhere (table entries at their +-254 extremes)."""
    N, K = 256, 2560
    W = si.weight(N, K, seed=9)
    x = torch.where(torch.arange(K) % 3 == 0, -1.0, 1.0).view(1, K).to(torch.bfloat16)
    g, codes, _ = oracle_weight(W)
    q_o, d_o, _ = oracle.quantize_act(x.float().numpy())
    assert np.abs(q_o).min() == 127
    acc_o = oracle.ternary_acc(codes, q_o)
    w = bl.pack(W.to(dev()))
    q, d, _ = bl.quantize_act(x.to(dev()))
    acc = torch.empty(1, N, dtype=torch.int32, device=dev())
    y = bl.lut_gemv(w, q, d, acc_dbg=acc)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    compare_outputs(y, oracle.rescale(acc_o, d_o, g))
