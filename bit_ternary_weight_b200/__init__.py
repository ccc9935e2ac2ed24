"""BitNet b1.58 BitLinear product on B200 (sm_100a): thin ctypes binding.

Every function here only checks and marshals torch tensors (device pointers,
sizes, dtypes and the current CUDA stream) into the C ABI of
``libbitlinear.so`` declared in ``include/bitlinear.h``; all arithmetic runs in
the library's CUDA kernels.  There is no CPU fallback: importing this package
fails if the library has not been built (``python
bit_ternary_weight_b200/build.py``), and every call raises ``BitLinearError`` on a
non-zero status.

Pages the operations follow (title, section):
  * "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete
    Guide", "Understanding the Two-Phase Architecture" -- INT8 activation
    quantisation in front of an INT8 x INT2 linear, called from Python through
    ctypes (section "Compiling the INT2 CUDA Kernel").
  * "bit-floor" README, "The core math" and "What's inside" -- integer inner
    product, final scale multiply, mean-abs (ternary) and absmax (binary)
    weight scales, XNOR / popcount binary GEMV.
  * "BitCompute: 1.58-bit LLM Execution Engine", "Usage" and "Future
    Roadmap" -- ``ternary_matmul(inputs, weights) -> [M, N]``; four weights
    per byte.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitlinear.so")

BL_OK = 0
BL_ERR_NULL = 1
BL_ERR_DTYPE = 2
BL_ERR_SHAPE = 3
BL_ERR_ALIGN = 4
BL_ERR_NOT_DEVICE_PTR = 5
BL_ERR_WORKSPACE = 6
BL_ERR_CUDA = 7
BL_ERR_TIMEOUT = 8
BL_ERR_UNSUPPORTED = 9

BL_F32 = 0
BL_BF16 = 1

GEMV_MAX_M = 16


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str | None = None):
        self.status = status
        msg = _lib.bitlinear_status_string(status).decode()
        if status == BL_ERR_CUDA:
            msg += " (" + _lib.bitlinear_last_cuda_error().decode() + ")"
        if detail:
            msg += f" ({detail})"
        super().__init__(f"{where}: {msg}")


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python bit_ternary_weight_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

_vp, _i64, _int, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SIGNATURES = {
    "bitlinear_status_string": (ctypes.c_char_p, [_int]),
    "bitlinear_last_cuda_error": (ctypes.c_char_p, []),
    "bitlinear_packed_bytes": (_sz, [_i64, _i64]),
    "bitlinear_pack_workspace_bytes": (_sz, [_i64, _i64]),
    "bitlinear_pack": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _vp, _sz, _vp]),
    "bitlinear_pack_noalloc": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _vp]),
    "bitlinear_quantize_act": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "bitlinear_gemv": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _int, _i64,
                              _vp, _vp]),
    "bitlinear_gemv_fused": (_int, [_vp, _vp, _i64, _i64, _vp, _int, _i64, _i64, _vp, _int,
                                    _i64, _vp, _vp]),
    "bitlinear_gemv_fused_multi": (_int, [_int, _vp, _vp, _vp, _i64, _vp, _int, _i64, _i64,
                                          _vp, _int, _vp, _vp, ctypes.c_uint, _vp]),
    "bitlinear_gemv_plan": (_int, [_int, _vp, _i64, _i64, _int, _int, ctypes.c_uint, _vp, _vp]),
    "bitlinear_rmsnorm_quantize_act": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _int,
                                              ctypes.c_float, _vp, _vp, _vp, _vp]),
    "bitlinear_rmsnorm_gemv_fused_multi": (_int, [_int, _vp, _vp, _vp, _i64, _vp, _int, _vp,
                                                  _int, ctypes.c_float, _vp, _int, _vp, _vp,
                                                  ctypes.c_uint, _vp]),
    "bitlinear_gemm_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "bitlinear_gemm": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _int, _i64,
                              _vp, _vp, _sz, _vp]),
    "bitlinear_binary_packed_bytes": (_sz, [_i64, _i64]),
    "bitlinear_binary_pack": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _vp]),
    "bitlinear_binary_gemv": (_int, [_vp, _vp, _i64, _i64, _vp, _int, _vp, _int, _vp, _vp]),
    "bitlinear_lut_gemv": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _int, _vp, _vp]),
    "bitlinear_bitplane_bytes": (_sz, [_i64, _i64]),
    "bitlinear_bitplane_pack": (_int, [_vp, _i64, _i64, _vp, _vp]),
    "bitlinear_bitplane_gemv": (_int, [_vp, _vp, _i64, _i64, _vp, _int, _vp, _int, _vp, _vp]),
    "bitlinear_last_device_status": (_int, [_vp]),
    "bitlinear_device_sm_count": (_int, []),
}
class ChainStepC(ctypes.Structure):
    """Mirror of bitlinear_chain_step (include/bitlinear.h)."""
    _fields_ = [("count", ctypes.c_int),
                ("packed", ctypes.c_void_p * 8),
                ("w_scale", ctypes.c_void_p * 8),
                ("N", ctypes.c_int64 * 8),
                ("y", ctypes.c_void_p * 8),
                ("acc_dbg", ctypes.c_void_p * 8),
                ("K", ctypes.c_int64),
                ("x", ctypes.c_void_p),
                ("xt", ctypes.c_int),
                ("yt", ctypes.c_int),
                ("norm", ctypes.c_int),
                ("gain", ctypes.c_void_p),
                ("gt", ctypes.c_int),
                ("eps", ctypes.c_float)]


_SIGNATURES.update({
    "bitlinear_decode_linear": (_int, [_int, _vp, _vp, _vp, _i64, _int, _vp, _int, _vp, _vp, _int,
                                       ctypes.c_float, _vp, _int, _vp, _vp, _vp, ctypes.c_uint,
                                       _vp]),
    "bitlinear_attention_decode": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int,
                                          ctypes.c_double, _vp, _vp, _vp, _sz, ctypes.c_uint,
                                          _vp]),
    "bitlinear_rope_table": (_int, [_int, _int, ctypes.c_double, _vp, _vp]),
    "bitlinear_attention_workspace_bytes": (_sz, [_int, _int, _int]),
    "bitlinear_position_advance": (_int, [_vp, _vp]),
    "bitlinear_probe_mma_i8": (_int, [_int, _vp, _int, _vp]),
    "bitlinear_probe_mma_i8_issue": (_int, [_int, _int, _int, _vp, _int, _vp]),
    "bitlinear_chain_plan_bytes": (_sz, [_int]),
    "bitlinear_chain_plan": (_int, [_int, ctypes.POINTER(ChainStepC), _vp, _sz, _vp]),
    "bitlinear_chain_run": (_int, [_vp, _int, _vp]),
    "bitlinear_chain_run_timeout_test": (_int, [_vp, _int, ctypes.c_uint64, _vp]),
})

for _name, (_res, _args) in _SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

lib = _lib  # the raw C ABI, for callers that marshal pointers themselves


def _check(status: int, where: str) -> None:
    if status != BL_OK:
        raise BitLinearError(status, where)


def _dt(t: torch.dtype) -> int:
    if t == torch.float32:
        return BL_F32
    if t == torch.bfloat16:
        return BL_BF16
    return -1


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    # a CPU tensor still goes to the library, which rejects host pointers
    dev = device if device.type == "cuda" else None
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _on(device: torch.device):
    """Make the tensors' GPU current for the call: the library launches on the
    current device and rejects memory of any other GPU."""
    if device.type == "cuda":
        return torch.cuda.device(device)
    return contextlib.nullcontext()


_FLOATS = (torch.float32, torch.bfloat16)
_I8 = (torch.int8,)
_I32 = (torch.int32,)
_U8 = (torch.uint8,)
_F32 = (torch.float32,)
_BF16 = (torch.bfloat16,)


def _fits(t, where: str, name: str, dtypes, rows: int, cols: int, ld: int | None = None):
    """Refuse, before the call, a caller buffer of another element type than
    the kernel reads or writes there, or one that does not hold the `rows` x
    `cols` elements the kernel addresses (row r at element r * ld, ld = cols
    unless given): the library sees only a pointer, so a short or mistyped
    buffer would be read or written out of its bounds."""
    if t is None:
        return
    if t.dtype not in dtypes:
        want = " or ".join(str(d).replace("torch.", "") for d in dtypes)
        raise BitLinearError(BL_ERR_DTYPE, where,
                             f"{name} is {str(t.dtype).replace('torch.', '')}, needs {want}")
    if rows < 1 or cols < 1:
        return                      # the library rejects the shape itself
    ld = cols if ld is None else ld
    if rows == 1:
        ok = t.numel() >= cols and (t.is_contiguous() or
                                    (t.size(-1) >= cols and t.stride(-1) == 1))
    elif t.dim() == 2:
        ok = (t.size(0) >= rows and t.size(1) >= cols and t.stride(0) == ld and
              (t.size(1) == 1 or t.stride(1) == 1))
    else:
        ok = t.dim() == 1 and t.is_contiguous() and ld == cols and t.numel() >= rows * cols
    esz = t.element_size()
    if ok:
        avail = t.untyped_storage().nbytes() - t.storage_offset() * esz
        ok = ((rows - 1) * ld + cols) * esz <= avail
    if not ok:
        pitch = f" with row pitch {ld}" if rows > 1 and ld != cols else ""
        raise BitLinearError(BL_ERR_SHAPE, where, f"{name} of shape {tuple(t.shape)} and strides "
                             f"{tuple(t.stride())} does not hold [{rows}][{cols}]{pitch}")


def _same_k(weights, where: str) -> int:
    """The shared K of products that read one activation row."""
    if not weights:
        raise BitLinearError(BL_ERR_SHAPE, where, "no weights")
    K = weights[0].K
    if any(w.K != K for w in weights):
        raise BitLinearError(BL_ERR_SHAPE, where,
                             f"weights of different K {sorted({w.K for w in weights})} share x")
    return K


def _per_product(lst, n: int, where: str, name: str):
    if lst is not None and len(lst) != n:
        raise BitLinearError(BL_ERR_SHAPE, where, f"{len(lst)} {name} for {n} weights")


def _same_dtype(outs, where: str):
    if any(o.dtype != outs[0].dtype for o in outs):
        raise BitLinearError(BL_ERR_DTYPE, where, "outputs of mixed element types")


def _weight(w, where: str):
    """The buffers of a packed ternary weight hold its N x K codes and gamma."""
    _fits(w.packed, where, "packed", _U8, 1, packed_bytes(w.N, w.K))
    _fits(w.w_scale, where, "w_scale", _F32, 1, 1)


def _act(x, where: str, K: int, name: str = "x"):
    """The activations of a product have the weight's K features."""
    if x.dim() == 0 or x.shape[-1] != K:
        raise BitLinearError(BL_ERR_SHAPE, where,
                             f"{name} of shape {tuple(x.shape)} for a weight of K={K}")


def _outputs(where: str, weights, outs, acc_dbgs, M: int, lds=None):
    """Products sharing one launch: an output (one element type for all) and
    an optional int32 accumulator per weight, each [M][N]."""
    n = len(weights)
    _per_product(outs, n, where, "outputs")
    _per_product(acc_dbgs, n, where, "accumulators")
    _same_dtype(outs, where)
    for i, w in enumerate(weights):
        _weight(w, where)
        _fits(outs[i], where, f"outs[{i}]", _FLOATS, M, w.N, None if lds is None else lds[i])
        _fits(None if acc_dbgs is None else acc_dbgs[i], where, f"acc_dbgs[{i}]", _I32, M, w.N)


def _one_token(where: str, w, x, xtypes, out, acc_dbg, name: str = "x"):
    """One token x [K] in, y [N] (and the int32 accumulators) out."""
    _act(x, where, w.K, name)
    _fits(x, where, name, xtypes, 1, w.K)
    _fits(out, where, "out", _FLOATS, 1, w.N)
    _fits(acc_dbg, where, "acc_dbg", _I32, 1, w.N)


def _pre_quantised(where: str, w, q, d, rowsum, M: int, out, acc_dbg):
    """The operands of a product on pre-quantised activations."""
    _weight(w, where)
    _act(q, where, w.K, "q")
    _fits(q, where, "q", _I8, M, w.K)
    _fits(d, where, "d", _F32, 1, M)
    _fits(rowsum, where, "rowsum", _I32, 1, M)
    _fits(out, where, "out", _FLOATS, M, w.N, out.stride(0))
    _fits(acc_dbg, where, "acc_dbg", _I32, M, w.N)


@dataclass
class TernaryWeight:
    """A packed ternary weight: TL bytes, the fp32 gamma_eff and the shape."""
    packed: torch.Tensor   # uint8 [bitlinear_packed_bytes(N, K)]
    w_scale: torch.Tensor  # float32 [1]
    N: int
    K: int


@dataclass
class BinaryWeight:
    bits: torch.Tensor     # int64 [N, K/64] (uint64 words)
    s_w: torch.Tensor      # float32 [1]
    N: int
    K: int


def packed_bytes(N: int, K: int) -> int:
    return int(_lib.bitlinear_packed_bytes(N, K))


def pack(W: torch.Tensor) -> TernaryWeight:
    """Absmean-quantise and 2-bit pack a weight [N, K] (fp32 or bf16, CUDA)."""
    W = W.contiguous()
    N, K = W.shape
    nbytes = packed_bytes(N, K)
    if nbytes == 0:
        raise BitLinearError(BL_ERR_SHAPE, "pack")
    packed = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    w_scale = torch.empty(1, dtype=torch.float32, device=W.device)
    ws_bytes = int(_lib.bitlinear_pack_workspace_bytes(N, K))
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=W.device)
    with _on(W.device):
        _check(_lib.bitlinear_pack(_ptr(W), _dt(W.dtype), N, K, _ptr(packed), _ptr(w_scale),
                                   _ptr(ws), ws.numel(), _stream(W.device)), "bitlinear_pack")
    return TernaryWeight(packed, w_scale, N, K)


PACK_NOALLOC_MAX_ROWS = 65536


def pack_noalloc(W: torch.Tensor, packed: torch.Tensor, w_scale: torch.Tensor) -> TernaryWeight:
    """Like ``pack`` but into caller-given buffers and with no workspace: the
    library keeps the scratch it needs in a device array of its own (N must
    not exceed PACK_NOALLOC_MAX_ROWS).  For callers that cannot allocate
    device memory when they pack; this function allocates nothing either."""
    N, K = W.shape
    where = "bitlinear_pack_noalloc"
    _fits(W, where, "W", _FLOATS, N, K)
    _fits(packed, where, "packed", _U8, 1, packed_bytes(N, K))
    _fits(w_scale, where, "w_scale", _F32, 1, 1)
    with _on(W.device):
        _check(_lib.bitlinear_pack_noalloc(_ptr(W), _dt(W.dtype), N, K, _ptr(packed),
                                           _ptr(w_scale), _stream(W.device)),
               "bitlinear_pack_noalloc")
    return TernaryWeight(packed, w_scale, N, K)


def quantize_act(x: torch.Tensor, out=None):
    """Per-token absmax int8: returns (q int8 [M,K], d fp32 [M], rowsum int32 [M]),
    written into out=(q, d, rowsum) when given."""
    if x.dim() == 1:
        x = x.unsqueeze(0)
    M, K = x.shape
    if out is None:
        q = torch.empty(M, K, dtype=torch.int8, device=x.device)
        d = torch.empty(M, dtype=torch.float32, device=x.device)
        r = torch.empty(M, dtype=torch.int32, device=x.device)
    else:
        q, d, r = out
    where = "bitlinear_quantize_act"
    _fits(x, where, "x", _FLOATS, M, K, x.stride(0))
    _fits(q, where, "q", _I8, M, K)
    _fits(d, where, "d", _F32, 1, M)
    _fits(r, where, "rowsum", _I32, 1, M)
    with _on(x.device):
        _check(_lib.bitlinear_quantize_act(_ptr(x), _dt(x.dtype), M, K, x.stride(0), _ptr(q),
                                           _ptr(d), _ptr(r), _stream(x.device)),
               "bitlinear_quantize_act")
    return q, d, r


def _out(M, N, out_dtype, device, out):
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=device)
    return out


def gemv(w: TernaryWeight, q, d, rowsum, out_dtype=torch.bfloat16, out=None, acc_dbg=None):
    """Decode GEMV (1 <= M <= 16) on pre-quantised activations."""
    M = q.shape[0]
    out = _out(M, w.N, out_dtype, q.device, out)
    _pre_quantised("bitlinear_gemv", w, q, d, rowsum, M, out, acc_dbg)
    with _on(q.device):
        _check(_lib.bitlinear_gemv(_ptr(w.packed), _ptr(w.w_scale), w.N, w.K, _ptr(q), _ptr(d),
                                   _ptr(rowsum), M, _ptr(out), _dt(out.dtype), out.stride(0),
                                   _ptr(acc_dbg), _stream(q.device)), "bitlinear_gemv")
    return out


def gemv_fused(w: TernaryWeight, x: torch.Tensor, out_dtype=torch.bfloat16, out=None,
               acc_dbg=None):
    """Decode BitLinear in one launch: quantise x, ternary GEMV, rescale (M <= 16)."""
    if x.dim() == 1:
        x = x.unsqueeze(0)
    M = x.shape[0]
    out = _out(M, w.N, out_dtype, x.device, out)
    where = "bitlinear_gemv_fused"
    _weight(w, where)
    _act(x, where, w.K)
    _fits(x, where, "x", _FLOATS, M, w.K, x.stride(0))
    _fits(out, where, "out", _FLOATS, M, w.N, out.stride(0))
    _fits(acc_dbg, where, "acc_dbg", _I32, M, w.N)
    with _on(x.device):
        _check(_lib.bitlinear_gemv_fused(_ptr(w.packed), _ptr(w.w_scale), w.N, w.K, _ptr(x),
                                         _dt(x.dtype), x.stride(0), M, _ptr(out), _dt(out.dtype),
                                         out.stride(0), _ptr(acc_dbg), _stream(x.device)),
               "bitlinear_gemv_fused")
    return out


GEMV_MAX_PROBLEMS = 8
BL_FLAG_PDL = 1
BL_FLAG_SMALL_BATCH_DP4A = 2
BL_FLAG_SMALL_BATCH_TENSOR = 4


_SMALL_BATCH = {"auto": 0, "dp4a": BL_FLAG_SMALL_BATCH_DP4A, "tensor": BL_FLAG_SMALL_BATCH_TENSOR}


def gemv_fused_multi(weights, x: torch.Tensor, out_dtype=torch.bfloat16, outs=None,
                     acc_dbgs=None, pdl: bool = False, small_batch: str = "auto"):
    """Several decode BitLinears sharing the activations x, in one launch.

    weights: list of TernaryWeight with the same K (q/k/v or gate/up of a layer).
    pdl: allow the launch to overlap the preceding kernel's tail (programmatic
    dependent launch); only when the weights were not written by that kernel.
    small_batch: for 2 .. 16 tokens, "auto" (the measured crossover), "dp4a"
    (the multi-token streaming kernel) or "tensor" (the tensor-core kernel),
    each where it applies; the results are identical.
    """
    if x.dim() == 1:
        x = x.unsqueeze(0)
    n = len(weights)
    M = x.shape[0]
    where = "bitlinear_gemv_fused_multi"
    K = _same_k(weights, where)
    if outs is None:
        outs = [torch.empty(M, w.N, dtype=out_dtype, device=x.device) for w in weights]
    _act(x, where, K)
    _fits(x, where, "x", _FLOATS, M, K, x.stride(0))
    _outputs(where, weights, outs, acc_dbgs, M, [o.stride(0) for o in outs])
    P = ctypes.c_void_p * n
    I64 = ctypes.c_int64 * n
    packed = P(*[w.packed.data_ptr() for w in weights])
    scales = P(*[w.w_scale.data_ptr() for w in weights])
    Ns = I64(*[w.N for w in weights])
    ys = P(*[o.data_ptr() for o in outs])
    ldys = I64(*[o.stride(0) for o in outs])
    accs = None if acc_dbgs is None else P(*[0 if a is None else a.data_ptr() for a in acc_dbgs])
    with _on(x.device):
        _check(_lib.bitlinear_gemv_fused_multi(n, packed, scales, Ns, weights[0].K, _ptr(x),
                                               _dt(x.dtype), x.stride(0), M, ys, _dt(outs[0].dtype),
                                               ldys, accs,
                                               (BL_FLAG_PDL if pdl else 0) | _SMALL_BATCH[small_batch],
                                               _stream(x.device)), "bitlinear_gemv_fused_multi")
    return outs


GEMV_KERNELS = {1: "stream", 2: "tensor", 3: "stream_mt", 4: "dp4a"}


def gemv_plan(Ns, K: int, M: int, xdtype=torch.bfloat16, fused: bool = True,
              small_batch: str = "auto"):
    """Which GEMV kernel gemv_fused_multi (fused) or gemv (pre-quantised) runs
    for these shapes on the current device: ("stream" | "tensor" | "stream_mt"
    | "dp4a", cluster size of the tensor-core kernel or 0)."""
    n = len(Ns)
    Narr = (ctypes.c_int64 * n)(*Ns)
    kern, cl = ctypes.c_int(0), ctypes.c_int(0)
    _check(_lib.bitlinear_gemv_plan(n, Narr, K, M, _dt(xdtype), 1 if fused else 0,
                                    _SMALL_BATCH[small_batch],
                                    ctypes.byref(kern), ctypes.byref(cl)), "bitlinear_gemv_plan")
    return GEMV_KERNELS[kern.value], cl.value


RMS_EPS = 1e-5  # default RMSNorm epsilon (the library's reading; the pages give none)


def rmsnorm_quantize_act(x: torch.Tensor, gain=None, eps: float = RMS_EPS, out=None):
    """RMSNorm each token (gain [K] fp32/bf16 or None), then per-token absmax
    int8: returns (q int8 [M,K], d fp32 [M], rowsum int32 [M])."""
    if x.dim() == 1:
        x = x.unsqueeze(0)
    M, K = x.shape
    if out is None:
        q = torch.empty(M, K, dtype=torch.int8, device=x.device)
        d = torch.empty(M, dtype=torch.float32, device=x.device)
        r = torch.empty(M, dtype=torch.int32, device=x.device)
    else:
        q, d, r = out
    gt = BL_F32 if gain is None else _dt(gain.dtype)
    where = "bitlinear_rmsnorm_quantize_act"
    _fits(x, where, "x", _FLOATS, M, K, x.stride(0))
    _fits(gain, where, "gain", _FLOATS, 1, K)
    _fits(q, where, "q", _I8, M, K)
    _fits(d, where, "d", _F32, 1, M)
    _fits(r, where, "rowsum", _I32, 1, M)
    with _on(x.device):
        _check(_lib.bitlinear_rmsnorm_quantize_act(_ptr(x), _dt(x.dtype), M, K, x.stride(0),
                                                   _ptr(gain), gt, float(eps), _ptr(q), _ptr(d),
                                                   _ptr(r), _stream(x.device)),
               "bitlinear_rmsnorm_quantize_act")
    return q, d, r


def rmsnorm_gemv_fused_multi(weights, x: torch.Tensor, gain=None, eps: float = RMS_EPS,
                             out_dtype=torch.bfloat16, outs=None, acc_dbgs=None,
                             pdl: bool = False):
    """One token through RMSNorm, quantisation and several decode BitLinears
    sharing it (gate/up, q/k/v), in one launch.  x: [K] or [1, K]."""
    x = x.reshape(-1)
    n = len(weights)
    where = "bitlinear_rmsnorm_gemv_fused_multi"
    K = _same_k(weights, where)
    if outs is None:
        outs = [torch.empty(1, w.N, dtype=out_dtype, device=x.device) for w in weights]
    _act(x, where, K)
    _fits(x, where, "x", _FLOATS, 1, K)
    _fits(gain, where, "gain", _FLOATS, 1, K)
    _outputs(where, weights, outs, acc_dbgs, 1)
    P = ctypes.c_void_p * n
    I64 = ctypes.c_int64 * n
    packed = P(*[w.packed.data_ptr() for w in weights])
    scales = P(*[w.w_scale.data_ptr() for w in weights])
    Ns = I64(*[w.N for w in weights])
    ys = P(*[o.data_ptr() for o in outs])
    ldys = I64(*[o.stride(0) if o.dim() > 1 else o.numel() for o in outs])
    accs = None if acc_dbgs is None else P(*[0 if a is None else a.data_ptr() for a in acc_dbgs])
    gt = BL_F32 if gain is None else _dt(gain.dtype)
    with _on(x.device):
        _check(_lib.bitlinear_rmsnorm_gemv_fused_multi(
            n, packed, scales, Ns, weights[0].K, _ptr(x), _dt(x.dtype), _ptr(gain), gt,
            float(eps), ys, _dt(outs[0].dtype), ldys, accs, BL_FLAG_PDL if pdl else 0,
            _stream(x.device)), "bitlinear_rmsnorm_gemv_fused_multi")
    return outs


BL_ACT_PLAIN = 0
BL_ACT_RMSNORM = 1
BL_ACT_RELU2_GATE = 2


def decode_linear(weights, x: torch.Tensor, act: int = BL_ACT_PLAIN, x2=None, gain=None,
                  eps: float = RMS_EPS, outs=None, resid=None, out_dtype=torch.bfloat16,
                  acc_dbgs=None, pdl: bool = False):
    """One token through a decoder layer's BitLinears sharing an input, in one
    launch: act (plain / RMSNorm with gain / squared-ReLU gate of x and x2),
    the products, the rescale and, per product, an optional residual
    (resid[i]: bf16 [N] added before the rounding; may be outs[i] itself)."""
    x = x.reshape(-1)
    n = len(weights)
    where = "bitlinear_decode_linear"
    K = _same_k(weights, where)
    if outs is None:
        outs = [torch.empty(w.N, dtype=out_dtype, device=x.device) for w in weights]
    _act(x, where, K)
    _fits(x, where, "x", _FLOATS, 1, K)
    if x2 is not None:
        _act(x2.reshape(-1), where, K, "x2")
        _fits(x2, where, "x2", _FLOATS, 1, K)
    _fits(gain, where, "gain", _FLOATS, 1, K)
    _outputs(where, weights, outs, acc_dbgs, 1)
    _per_product(resid, n, where, "residuals")
    for i, w in enumerate(weights):
        _fits(None if resid is None else resid[i], where, f"resid[{i}]", _BF16, 1, w.N)
    P = ctypes.c_void_p * n
    I64 = ctypes.c_int64 * n
    packed = P(*[w.packed.data_ptr() for w in weights])
    scales = P(*[w.w_scale.data_ptr() for w in weights])
    Ns = I64(*[w.N for w in weights])
    ys = P(*[o.data_ptr() for o in outs])
    ldys = I64(*[w.N for w in weights])
    res = None if resid is None else P(*[0 if r is None else r.data_ptr() for r in resid])
    accs = None if acc_dbgs is None else P(*[0 if a is None else a.data_ptr() for a in acc_dbgs])
    gt = BL_F32 if gain is None else _dt(gain.dtype)
    with _on(x.device):
        _check(_lib.bitlinear_decode_linear(
            n, packed, scales, Ns, weights[0].K, act, _ptr(x), _dt(x.dtype), _ptr(x2), _ptr(gain),
            gt, float(eps), ys, _dt(outs[0].dtype), ldys, res, accs, BL_FLAG_PDL if pdl else 0,
            _stream(x.device)), "bitlinear_decode_linear")
    return outs


def attention_workspace(H: int, Hkv: int, T_max: int, device) -> torch.Tensor:
    """A zeroed workspace for attention_decode (reusable by ordered calls)."""
    n = int(_lib.bitlinear_attention_workspace_bytes(H, Hkv, T_max))
    if n == 0:
        raise BitLinearError(BL_ERR_SHAPE, "bitlinear_attention_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def rope_table(T_max: int, rope_base: float = 10000.0, device="cuda") -> torch.Tensor:
    """(cos, sin) of every (position, pair) angle, fp32 [T_max, 64, 2]."""
    tab = torch.empty(T_max, 64, 2, dtype=torch.float32, device=device)
    with _on(tab.device):
        _check(_lib.bitlinear_rope_table(128, T_max, float(rope_base), _ptr(tab),
                                         _stream(tab.device)), "bitlinear_rope_table")
    return tab


def attention_decode(q, k, v, cache_k, cache_v, pos, H: int, Hkv: int, out=None,
                     rope_base: float = 10000.0, workspace=None, table=None, pdl: bool = False):
    """One token's attention with RoPE over a bf16 cache [Hkv, T_max, 128];
    pos: int32 device scalar (this token's position; the cache row written)."""
    D = 128
    T_max = cache_k.shape[-2]
    if out is None:
        out = torch.empty(H * D, dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        workspace = attention_workspace(H, Hkv, T_max, q.device)
    where = "bitlinear_attention_decode"
    _fits(q, where, "q", _BF16, 1, H * D)
    _fits(k, where, "k", _BF16, 1, Hkv * D)
    _fits(v, where, "v", _BF16, 1, Hkv * D)
    _fits(cache_k, where, "cache_k", _BF16, 1, Hkv * T_max * D)
    _fits(cache_v, where, "cache_v", _BF16, 1, Hkv * T_max * D)
    _fits(pos, where, "pos", _I32, 1, 1)
    _fits(out, where, "out", _BF16, 1, H * D)
    _fits(table, where, "table", _F32, 1, T_max * D)
    _fits(workspace, where, "workspace", (workspace.dtype,), 1, workspace.numel())
    ws_bytes = workspace.numel() * workspace.element_size()
    with _on(q.device):
        _check(_lib.bitlinear_attention_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(cache_k),
                                               _ptr(cache_v), _ptr(pos), H, Hkv, D, T_max,
                                               float(rope_base), _ptr(table), _ptr(out),
                                               _ptr(workspace), ws_bytes,
                                               BL_FLAG_PDL if pdl else 0,
                                               _stream(q.device)),
               "bitlinear_attention_decode")
    return out


def position_advance(pos: torch.Tensor):
    _fits(pos, "bitlinear_position_advance", "pos", _I32, 1, 1)
    with _on(pos.device):
        _check(_lib.bitlinear_position_advance(_ptr(pos), _stream(pos.device)),
               "bitlinear_position_advance")


@dataclass
class ChainStep:
    """One step of a decode chain: products sharing the token x (1 .. 8 weights
    with the same K), each written to its output [N] (or [1, N]); RMSNorm in
    front when `norm` or a gain is given."""
    weights: list
    x: torch.Tensor
    outs: list
    norm: bool = False
    gain: torch.Tensor | None = None
    eps: float = RMS_EPS
    acc_dbgs: list | None = None


class DecodeChain:
    """A token's chain of dependent decode BitLinears run as ONE persistent
    launch (bitlinear_chain_plan / bitlinear_chain_run).  The plan lives in a
    device buffer owned by this object; the tensors the steps name must stay
    alive and in place while the chain is used."""

    def __init__(self, steps, device=None):
        n = len(steps)
        device = device or steps[0].x.device
        arr = (ChainStepC * n)()
        for i, st in enumerate(steps):
            where = f"bitlinear_chain_plan (step {i})"
            K = _same_k(st.weights, where)
            _act(st.x, where, K)
            _fits(st.x, where, "x", _FLOATS, 1, K)
            _fits(st.gain, where, "gain", _FLOATS, 1, K)
            _outputs(where, st.weights, st.outs, st.acc_dbgs, 1)
            c = arr[i]
            c.count = len(st.weights)
            for j, (w, o) in enumerate(zip(st.weights, st.outs)):
                c.packed[j] = w.packed.data_ptr()
                c.w_scale[j] = w.w_scale.data_ptr()
                c.N[j] = w.N
                c.y[j] = o.data_ptr()
                a = None if st.acc_dbgs is None else st.acc_dbgs[j]
                c.acc_dbg[j] = 0 if a is None else a.data_ptr()
            c.K = st.weights[0].K
            c.x = st.x.data_ptr()
            c.xt = _dt(st.x.dtype)
            c.yt = _dt(st.outs[0].dtype)
            c.norm = 1 if (st.norm or st.gain is not None) else 0
            c.gain = 0 if st.gain is None else st.gain.data_ptr()
            c.gt = BL_F32 if st.gain is None else _dt(st.gain.dtype)
            c.eps = float(st.eps)
        nbytes = int(_lib.bitlinear_chain_plan_bytes(n))
        if nbytes == 0:
            raise BitLinearError(BL_ERR_SHAPE, "bitlinear_chain_plan_bytes")
        self.n = n
        self.steps = steps
        self.device = torch.device(device)
        self.plan = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        with _on(self.device):
            _check(_lib.bitlinear_chain_plan(n, arr, _ptr(self.plan), nbytes,
                                             _stream(self.device)), "bitlinear_chain_plan")
            torch.cuda.current_stream(self.device).synchronize()

    def run(self):
        with _on(self.device):
            _check(_lib.bitlinear_chain_run(_ptr(self.plan), self.n, _stream(self.device)),
                   "bitlinear_chain_run")

    def run_timeout_test(self, wait_limit_ns: int = 1_000_000):
        """Run with a wait that cannot complete (testing the timeout path)."""
        with _on(self.device):
            _check(_lib.bitlinear_chain_run_timeout_test(_ptr(self.plan), self.n, wait_limit_ns,
                                                         _stream(self.device)),
                   "bitlinear_chain_run_timeout_test")


def gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.bitlinear_gemm_workspace_bytes(M, N, K))


def gemm(w: TernaryWeight, q, d, rowsum, out_dtype=torch.bfloat16, out=None, acc_dbg=None,
         workspace=None):
    """Prefill GEMM (any M) on the tcgen05 int8 tensor cores."""
    M = q.shape[0]
    out = _out(M, w.N, out_dtype, q.device, out)
    need = gemm_workspace_bytes(M, w.N, w.K)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        # zero before its first use; every call leaves it zero again
        workspace = torch.zeros(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    where = "bitlinear_gemm"
    _pre_quantised(where, w, q, d, rowsum, M, out, acc_dbg)
    if workspace is not None:
        _fits(workspace, where, "workspace", (workspace.dtype,), 1, workspace.numel())
    with _on(q.device):
        _check(_lib.bitlinear_gemm(_ptr(w.packed), _ptr(w.w_scale), w.N, w.K, _ptr(q), _ptr(d),
                                   _ptr(rowsum), M, _ptr(out), _dt(out.dtype), out.stride(0),
                                   _ptr(acc_dbg), _ptr(workspace), ws_bytes, _stream(q.device)),
               "bitlinear_gemm")
    return out


GEMV_FUSED_MAX_M = 8          # up to here the fused GEMV kernels are always the faster path


def fused_gemv_preferred(M: int, N: int, K: int) -> bool:
    """Whether the fused GEMV beats quantise + tensor-core GEMM for M tokens:
    up to 8 tokens always; 9 .. 16 tokens where the small-batch tensor-core
    or multi-token streaming kernel takes the shape (measured on B200: both
    under the GEMM's ~11-13 us there), not the per-warp dp4a kernel."""
    if M * K > 163840 or M > 16:
        return False
    if M <= GEMV_FUSED_MAX_M:
        return True
    return gemv_plan([N], K, M)[0] in ("tensor", "stream_mt")


def linear(w: TernaryWeight, x: torch.Tensor, out_dtype=torch.bfloat16):
    """y = BitLinear(x): the fused dp4a GEMV for few tokens (see
    fused_gemv_preferred), else quantise + tensor-core GEMM."""
    x2 = x.reshape(-1, x.shape[-1])
    if fused_gemv_preferred(x2.shape[0], w.N, w.K):
        y = gemv_fused(w, x2, out_dtype)
    else:
        q, d, r = quantize_act(x2)
        y = gemm(w, q, d, r, out_dtype)
    return y.reshape(*x.shape[:-1], w.N)


def binary_pack(W: torch.Tensor) -> BinaryWeight:
    W = W.contiguous()
    N, K = W.shape
    nbytes = int(_lib.bitlinear_binary_packed_bytes(N, K))
    if nbytes == 0:
        raise BitLinearError(BL_ERR_SHAPE, "binary_pack")
    bits = torch.empty(N, K // 64, dtype=torch.int64, device=W.device)
    s_w = torch.empty(1, dtype=torch.float32, device=W.device)
    with _on(W.device):
        _check(_lib.bitlinear_binary_pack(_ptr(W), _dt(W.dtype), N, K, _ptr(bits), _ptr(s_w),
                                          _stream(W.device)), "bitlinear_binary_pack")
    return BinaryWeight(bits, s_w, N, K)


def binary_gemv(w: BinaryWeight, x: torch.Tensor, out_dtype=torch.bfloat16, out=None,
                acc_dbg=None):
    x = x.reshape(-1)
    if out is None:
        out = torch.empty(w.N, dtype=out_dtype, device=x.device)
    where = "bitlinear_binary_gemv"
    _fits(w.bits, where, "bits", (torch.int64,), 1, w.N * (w.K // 64))
    _fits(w.s_w, where, "s_w", _F32, 1, 1)
    _one_token(where, w, x, _FLOATS, out, acc_dbg)
    with _on(x.device):
        _check(_lib.bitlinear_binary_gemv(_ptr(w.bits), _ptr(w.s_w), w.N, w.K, _ptr(x),
                                          _dt(x.dtype), _ptr(out), _dt(out.dtype), _ptr(acc_dbg),
                                          _stream(x.device)), "bitlinear_binary_gemv")
    return out


def lut_gemv(w: TernaryWeight, q, d, out_dtype=torch.bfloat16, out=None, acc_dbg=None):
    """One token's ternary GEMV by table lookup (K <= 12288), on pre-quantised
    activations (q [1, K] or [K], d [1]); same results as gemv()."""
    q = q.reshape(-1)
    if out is None:
        out = torch.empty(1, w.N, dtype=out_dtype, device=q.device)
    where = "bitlinear_lut_gemv"
    _weight(w, where)
    _one_token(where, w, q, _I8, out, acc_dbg, "q")
    _fits(d, where, "d", _F32, 1, 1)
    with _on(q.device):
        _check(_lib.bitlinear_lut_gemv(_ptr(w.packed), _ptr(w.w_scale), w.N, w.K, _ptr(q),
                                       _ptr(d), _ptr(out), _dt(out.dtype), _ptr(acc_dbg),
                                       _stream(q.device)), "bitlinear_lut_gemv")
    return out


@dataclass
class BitPlaneWeight:
    """Ternary weight as (mag, sign) bit-planes, with the packed weight's gamma."""
    planes: torch.Tensor   # int64 [N, K/64, 2] (uint64 words)
    w_scale: torch.Tensor  # float32 [1]
    N: int
    K: int


def bitplane_pack(w: TernaryWeight) -> BitPlaneWeight:
    """Bit-planes of a packed ternary weight (same codes, same gamma)."""
    _weight(w, "bitlinear_bitplane_pack")
    planes = torch.empty(w.N, w.K // 64, 2, dtype=torch.int64, device=w.packed.device)
    with _on(w.packed.device):
        _check(_lib.bitlinear_bitplane_pack(_ptr(w.packed), w.N, w.K, _ptr(planes),
                                            _stream(w.packed.device)), "bitlinear_bitplane_pack")
    return BitPlaneWeight(planes, w.w_scale, w.N, w.K)


def bitplane_gemv(w: BitPlaneWeight, x: torch.Tensor, out_dtype=torch.bfloat16, out=None,
                  acc_dbg=None):
    """Ternary weights x the sign bits of one token: y = dot * (gamma * max|x|)."""
    x = x.reshape(-1)
    if out is None:
        out = torch.empty(w.N, dtype=out_dtype, device=x.device)
    where = "bitlinear_bitplane_gemv"
    _fits(w.planes, where, "planes", (torch.int64,), 1, w.N * (w.K // 64) * 2)
    _fits(w.w_scale, where, "w_scale", _F32, 1, 1)
    _one_token(where, w, x, _FLOATS, out, acc_dbg)
    with _on(x.device):
        _check(_lib.bitlinear_bitplane_gemv(_ptr(w.planes), _ptr(w.w_scale), w.N, w.K, _ptr(x),
                                            _dt(x.dtype), _ptr(out), _dt(out.dtype),
                                            _ptr(acc_dbg), _stream(x.device)),
               "bitlinear_bitplane_gemv")
    return out


def probe_mma_i8(reps: int = 4000, device="cuda", n: int = 128, issuers: int = 1) -> dict:
    """Time back-to-back tcgen05 int8 MMAs (128 x n x 32, A in tensor memory,
    B in shared memory, no operand traffic) on every SM from `issuers` warps
    at once: MAC per clock per SM and TOPS over the grid.  n = 128 with one
    issuer is the prefill GEMM's form."""
    dev = torch.device(device)
    grid = sm_count()
    out = torch.zeros(2 * issuers * grid, dtype=torch.int64, device=dev)
    with _on(dev):
        if n == 128 and issuers == 1:
            _check(_lib.bitlinear_probe_mma_i8(reps, _ptr(out), grid, _stream(dev)), "bitlinear_probe_mma_i8")
        else:
            _check(_lib.bitlinear_probe_mma_i8_issue(n, issuers, reps, _ptr(out), grid, _stream(dev)),
                   "bitlinear_probe_mma_i8_issue")
        torch.cuda.synchronize(dev)
    res = out.view(grid, issuers, 2).cpu()
    if bool((res < 0).any()):
        raise BitLinearError(BL_ERR_TIMEOUT, "bitlinear_probe_mma_i8")
    macs = float(reps) * 8 * 128 * n * 32            # per issuer
    cyc = res[:, :, 0].double().max(dim=1).values      # per CTA: its slowest issuer
    ns = res[:, :, 1].double()
    return {"reps": reps, "ctas": grid, "n": n, "issuers": issuers,
            "mac_per_clk_per_sm": float((issuers * macs / cyc).median()),
            "cycles_per_mma_per_sm": float((cyc / (reps * 8 * issuers)).median()),
            "tops": float(2 * issuers * macs * grid / ns.max() / 1e3),
            "ns_max": float(ns.max()), "cycles_median": float(cyc.median())}


def last_device_status(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(_lib.bitlinear_last_device_status(ctypes.c_void_p(s.cuda_stream)))


def sm_count() -> int:
    return int(_lib.bitlinear_device_sm_count())
