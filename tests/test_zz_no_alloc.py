"""bitlinear_pack_noalloc: packing for callers that cannot allocate device memory.

Some callers have no device allocator at hand when they pack weights (a plain
C host linking the library, or a runtime whose memory pool owns the GPU), so
this entry point takes no workspace and keeps its scratch in a device array of
its own.  Its results must equal those of bitlinear_pack, call after call.
This file is collected last on purpose: it also runs correctly on its own in a
fresh process, where its first call does the per-device set-up.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth_inputs as si


@pytest.fixture(scope="module")
def bl():
    import bit_ternary_weight_b200 as b
    return b


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_rejects_bad_arguments_before_any_cuda_call(bl):
    A = 0x7f0000000000
    L = bl.lib
    assert L.bitlinear_pack_noalloc(None, 0, 8, 64, A, A, None) == bl.BL_ERR_NULL
    assert L.bitlinear_pack_noalloc(A, 4, 8, 64, A, A, None) == bl.BL_ERR_DTYPE
    assert L.bitlinear_pack_noalloc(A, 0, bl.PACK_NOALLOC_MAX_ROWS + 1, 64, A, A,
                                    None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_pack_noalloc(A, 0, 8, 96, A, A, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_pack_noalloc(A + 4, 0, 8, 64, A, A, None) == bl.BL_ERR_ALIGN


@pytest.mark.gpu
def test_noalloc_matches_pack_on_consecutive_calls(bl):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    # two calls in a row; the second is smaller, so stale scratch from the
    # first call would show up if anything depended on it
    for (N, K, wdtype, seed) in [(6912, 2560, torch.float32, 21), (640, 2560, torch.bfloat16, 22)]:
        W = si.weight(N, K, seed=seed).to(wdtype).to(dev)
        nbytes = bl.packed_bytes(N, K)
        ref = bl.pack(W)
        packed = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        scale = torch.empty(1, dtype=torch.float32, device=dev)
        st = bl.lib.bitlinear_pack_noalloc(_p(W), bl.BL_F32 if wdtype == torch.float32 else bl.BL_BF16,
                                           N, K, _p(packed), _p(scale), stream)
        assert st == bl.BL_OK, bl.lib.bitlinear_status_string(st)
        torch.cuda.synchronize()
        # integer bytes and the fp32 scale's bit pattern: exact, like every
        # other packer check in this suite
        np.testing.assert_array_equal(packed.cpu().numpy(), ref.packed.cpu().numpy())
        assert scale.cpu().numpy().view(np.uint32)[0] == ref.w_scale.cpu().numpy().view(np.uint32)[0]
    assert bl.last_device_status() == bl.BL_OK
