"""Host-side checks of the Python binding's own argument checks (no GPU).

The library takes raw pointers, so it cannot see a short output, an
accumulator of another element type or an activation row with a stride: a
kernel would read or write past such a buffer.  The binding refuses them
with BL_ERR_SHAPE / BL_ERR_DTYPE before the library is called.  Layouts that
are valid (row-pitched output views, one-token vectors, views into one flat
buffer, a row shard of a packed weight, an in-place residual) pass the
binding and reach the library, which on CPU tensors answers with its own
device error (no GPU here, or memory that is not a GPU's), never with a
shape or type error.
"""
import ctypes

import pytest
import torch

BF16, F32, I8, I32 = torch.bfloat16, torch.float32, torch.int8, torch.int32

# size queries the binding may make before it refuses a call
_QUERIES = {"bitlinear_status_string", "bitlinear_last_cuda_error", "bitlinear_packed_bytes",
            "bitlinear_pack_workspace_bytes", "bitlinear_gemm_workspace_bytes",
            "bitlinear_binary_packed_bytes", "bitlinear_bitplane_bytes",
            "bitlinear_attention_workspace_bytes", "bitlinear_chain_plan_bytes"}


class _Spy:
    """The real library, recording every call that is not a size query."""

    def __init__(self, lib):
        self._lib = lib
        self.calls = []

    def __getattr__(self, name):
        fn = getattr(self._lib, name)
        if name in _QUERIES:
            return fn

        def call(*a):
            self.calls.append(name)
            return fn(*a)
        return call


@pytest.fixture()
def spy(monkeypatch):
    """The library behind the binding, recording its calls; CPU tensors have
    no CUDA stream to look up, so the library gets the null stream."""
    import bit_ternary_weight_b200 as b
    monkeypatch.setattr(b, "_stream", lambda device: ctypes.c_void_p(0))
    sp = _Spy(b._lib)
    monkeypatch.setattr(b, "_lib", sp)
    return sp


@pytest.fixture()
def bl(spy):
    import bit_ternary_weight_b200 as b
    return b


def _passes(bl, spy, fn):
    """The binding lets the call through: the library answers for the device."""
    spy.calls.clear()
    with pytest.raises(bl.BitLinearError) as e:
        fn()
    assert e.value.status in (bl.BL_ERR_NOT_DEVICE_PTR, bl.BL_ERR_CUDA,
                              bl.BL_ERR_UNSUPPORTED), str(e.value)
    assert spy.calls, "the library was not called"


def _refused(bl, spy, fn, status, words):
    spy.calls.clear()
    with pytest.raises(bl.BitLinearError) as e:
        fn()
    assert e.value.status == status, str(e.value)
    assert words in str(e.value), str(e.value)
    assert not spy.calls, f"the library was called: {spy.calls}"


def _weight(bl, N, K):
    return bl.TernaryWeight(torch.zeros(bl.packed_bytes(N, K), dtype=torch.uint8),
                            torch.ones(1, dtype=F32), N, K)


# ------------------------------------------------------------ valid layouts


def test_row_pitched_output_and_accumulators_pass(bl, spy):
    M, N, K = 4, 40, 256
    w = _weight(bl, N, K)
    big = torch.zeros(M, N + 24, dtype=BF16)
    acc = torch.zeros(M, N, dtype=I32)
    _passes(bl, spy, lambda: bl.gemv_fused(w, torch.zeros(M, K, dtype=BF16), out=big[:, :N],
                                           acc_dbg=acc))


def test_outputs_in_one_flat_buffer_pass(bl, spy):
    K = 256
    ws = [_weight(bl, N, K) for N in (64, 16, 16)]
    flat = torch.zeros(96, dtype=BF16)
    outs, off = [], 0
    for w in ws:
        outs.append(flat[off:off + w.N].view(1, w.N))
        off += w.N
    _passes(bl, spy, lambda: bl.gemv_fused_multi(ws, torch.zeros(1, K, dtype=BF16), outs=outs))


def test_row_shard_of_a_packed_weight_passes(bl, spy):
    from bit_ternary_weight_b200.sharding import row_partition, shard_weight
    w = _weight(bl, 100, 512)
    for sh in row_partition(100, 3):
        part = shard_weight(w, sh)
        y = torch.zeros(1, sh.rows, dtype=BF16)
        _passes(bl, spy, lambda: bl.gemv_fused_multi([part], torch.zeros(1, 512, dtype=BF16),
                                                     outs=[y]))


def test_pre_quantised_paths_pass(bl, spy):
    M, N, K = 3, 24, 192
    w = _weight(bl, N, K)
    x = torch.zeros(M, K, dtype=F32)
    q, d, r = torch.zeros(M, K, dtype=I8), torch.zeros(M, dtype=F32), torch.zeros(M, dtype=I32)
    _passes(bl, spy, lambda: bl.quantize_act(x, out=(q, d, r)))
    _passes(bl, spy, lambda: bl.gemv(w, q, d, r, acc_dbg=torch.zeros(M, N, dtype=I32)))
    _passes(bl, spy, lambda: bl.gemm(w, q, d, r, out=torch.zeros(M, N, dtype=F32)))
    _passes(bl, spy, lambda: bl.lut_gemv(w, q[:1], d[:1], acc_dbg=torch.zeros(N, dtype=I32)))


def test_one_token_decoder_calls_pass(bl, spy):
    K, N = 256, 256
    w = _weight(bl, N, K)
    h = torch.zeros(N, dtype=BF16)
    _passes(bl, spy, lambda: bl.decode_linear([w], torch.zeros(K, dtype=BF16), bl.BL_ACT_PLAIN,
                                              outs=[h], resid=[h]))
    H, Hkv, D, T = 4, 2, 128, 16
    x = torch.zeros(H * D, dtype=BF16)
    ck = torch.zeros(Hkv, T, D, dtype=BF16)
    cv = torch.zeros(Hkv, T, D, dtype=BF16)
    pos = torch.zeros(1, dtype=I32)
    _passes(bl, spy, lambda: bl.attention_decode(x, x[:Hkv * D], x[:Hkv * D], ck, cv, pos, H, Hkv))


# ------------------------------------------------------------ refused buffers


def test_accumulator_of_another_type_is_refused(bl, spy):
    w = _weight(bl, 16, 64)
    q, d, r = torch.zeros(1, 64, dtype=I8), torch.zeros(1, dtype=F32), torch.zeros(1, dtype=I32)
    _refused(bl, spy, lambda: bl.gemv(w, q, d, r, acc_dbg=torch.zeros(1, 16, dtype=torch.int16)),
             bl.BL_ERR_DTYPE, "acc_dbg is int16")


def test_short_output_is_refused(bl, spy):
    w = _weight(bl, 16, 64)
    x = torch.zeros(2, 64, dtype=BF16)
    _refused(bl, spy, lambda: bl.gemv_fused(w, x, out=torch.zeros(2, 8, dtype=BF16)),
             bl.BL_ERR_SHAPE, "out of shape (2, 8)")
    _refused(bl, spy, lambda: bl.gemv_fused(w, x, out=torch.zeros(1, 16, dtype=BF16)),
             bl.BL_ERR_SHAPE, "does not hold [2][16]")
    _refused(bl, spy, lambda: bl.gemv_fused(w, x, acc_dbg=torch.zeros(2, 15, dtype=I32)),
             bl.BL_ERR_SHAPE, "acc_dbg")


def test_activations_of_another_width_or_stride_are_refused(bl, spy):
    w = _weight(bl, 16, 128)
    _refused(bl, spy, lambda: bl.gemv_fused(w, torch.zeros(1, 192, dtype=BF16)),
             bl.BL_ERR_SHAPE, "for a weight of K=128")
    strided = torch.zeros(2, 256, dtype=BF16)[:, ::2]
    _refused(bl, spy, lambda: bl.gemv_fused(w, strided), bl.BL_ERR_SHAPE, "x of shape (2, 128)")
    q = torch.zeros(2, 192, dtype=I8)[:, :128]       # rows 192 apart, not K
    d, r = torch.zeros(2, dtype=F32), torch.zeros(2, dtype=I32)
    _refused(bl, spy, lambda: bl.gemv(w, q, d, r), bl.BL_ERR_SHAPE, "q of shape (2, 128)")
    _refused(bl, spy, lambda: bl.gemv(w, q.contiguous(), d[:1], r), bl.BL_ERR_SHAPE, "d of shape")
    _refused(bl, spy, lambda: bl.binary_gemv(bl.BinaryWeight(torch.zeros(16, 2, dtype=torch.int64),
                                                              torch.ones(1), 16, 128),
                                             torch.zeros(64, dtype=BF16)),
             bl.BL_ERR_SHAPE, "for a weight of K=128")


def test_products_that_cannot_share_a_launch_are_refused(bl, spy):
    x = torch.zeros(1, 256, dtype=BF16)
    a, b = _weight(bl, 16, 256), _weight(bl, 16, 512)
    _refused(bl, spy, lambda: bl.gemv_fused_multi([a, b], x), bl.BL_ERR_SHAPE, "different K")
    c = _weight(bl, 32, 256)
    _refused(bl, spy, lambda: bl.gemv_fused_multi([a, c], x, outs=[torch.zeros(1, 16, dtype=BF16)]),
             bl.BL_ERR_SHAPE, "1 outputs for 2 weights")
    _refused(bl, spy, lambda: bl.gemv_fused_multi(
        [a, c], x, outs=[torch.zeros(1, 16, dtype=BF16), torch.zeros(1, 32, dtype=F32)]),
        bl.BL_ERR_DTYPE, "mixed element types")
    _refused(bl, spy, lambda: bl.gemv_fused_multi([], x), bl.BL_ERR_SHAPE, "no weights")


def test_short_packed_weight_is_refused(bl, spy):
    w = bl.TernaryWeight(torch.zeros(bl.packed_bytes(16, 256) - 16, dtype=torch.uint8),
                         torch.ones(1), 16, 256)
    _refused(bl, spy, lambda: bl.gemv_fused(w, torch.zeros(1, 256, dtype=BF16)),
             bl.BL_ERR_SHAPE, "packed of shape")


def test_pack_noalloc_needs_row_major_weights_and_room(bl, spy):
    W = torch.zeros(64, 16, dtype=F32).t()              # [16, 64] seen through a transpose
    packed = torch.zeros(bl.packed_bytes(16, 64), dtype=torch.uint8)
    _refused(bl, spy, lambda: bl.pack_noalloc(W, packed, torch.zeros(1)), bl.BL_ERR_SHAPE, "W of shape")
    _refused(bl, spy, lambda: bl.pack_noalloc(W.contiguous(), packed[:-1], torch.zeros(1)),
             bl.BL_ERR_SHAPE, "packed of shape")
    _refused(bl, spy, lambda: bl.pack_noalloc(W.contiguous(), packed, torch.zeros(1, dtype=BF16)),
             bl.BL_ERR_DTYPE, "w_scale is bfloat16")


def test_attention_buffers_are_checked(bl, spy):
    H, Hkv, D, T = 4, 2, 128, 16
    x = torch.zeros(H * D, dtype=BF16)
    ck = torch.zeros(Hkv, T, D, dtype=BF16)
    _refused(bl, spy, lambda: bl.attention_decode(x, x[:Hkv * D], x[:Hkv * D], ck, ck[:1],
                                                  torch.zeros(1, dtype=I32), H, Hkv),
             bl.BL_ERR_SHAPE, "cache_v")
    _refused(bl, spy, lambda: bl.attention_decode(x, x[:Hkv * D], x[:Hkv * D], ck, ck,
                                                  torch.zeros(1, dtype=torch.int64), H, Hkv),
             bl.BL_ERR_DTYPE, "pos is int64")
    _refused(bl, spy, lambda: bl.attention_decode(x[:D], x[:Hkv * D], x[:Hkv * D], ck, ck,
                                                  torch.zeros(1, dtype=I32), H, Hkv),
             bl.BL_ERR_SHAPE, "q of shape (128,)")


def test_decoder_residual_and_chain_steps_are_checked(bl, spy):
    w = _weight(bl, 256, 256)
    x = torch.zeros(256, dtype=BF16)
    _refused(bl, spy, lambda: bl.decode_linear([w], x, bl.BL_ACT_PLAIN,
                                               resid=[torch.zeros(256, dtype=F32)]),
             bl.BL_ERR_DTYPE, "resid[0] is float32")
    step = bl.ChainStep([w], x, [torch.zeros(1, 256, dtype=BF16)],
                        acc_dbgs=[torch.zeros(256, dtype=torch.int64)])
    _refused(bl, spy, lambda: bl.DecodeChain([step], device="cpu"), bl.BL_ERR_DTYPE,
             "acc_dbgs[0] is int64")
    step = bl.ChainStep([w], torch.zeros(128, dtype=BF16), [torch.zeros(1, 256, dtype=BF16)])
    _refused(bl, spy, lambda: bl.DecodeChain([step], device="cpu"), bl.BL_ERR_SHAPE, "step 0")
