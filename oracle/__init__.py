"""CPU oracle for the BitNet b1.58 BitLinear product -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The CUDA library never does, and
this package imports nothing from it.

The arithmetic lives in ``bitlinear_oracle.c`` (plain C loops, fp64 weight-scale
sum, fp32 decisions, exact integer products); this module only compiles it
with gcc on first use and marshals numpy arrays through ctypes.  The header of
the C file lists the pages and sections each function follows and the reading
taken where the pages are silent.

Pins (tests/test_oracle_pins.py) tie every function to something other than
itself: a hand-worked 4x4 example, brute-force fp64 matmul of the dequantised
operands, invariants (code alphabet, |q| <= 127, the Gaussian zero fraction,
the XNOR/popcount identity, permutation invariance) and hand-written layout
fixtures.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitlinear_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
# The test of the pins themselves (tests/test_oracle_mutations.py) builds
# copies of the C source with one planted mistake each and points the oracle
# at such a copy through this variable; nothing else sets it.
_LIB_OVERRIDE = os.environ.get("BITLINEAR_ORACLE_LIB")
_lock = threading.Lock()
_lib = None

_CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-shared", "-fPIC", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile the oracle C source into ``liboracle.so`` next to it (or, under
    BITLINEAR_ORACLE_LIB, return that prebuilt library untouched)."""
    if _LIB_OVERRIDE:
        return _LIB_OVERRIDE
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        i64, f32, vp = ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
        sig = {
            "oracle_weight_scale": (f32, [vp, i64, i64]),
            "oracle_ternary_codes": (None, [vp, i64, i64, f32, vp]),
            "oracle_packed_bytes": (i64, [i64, i64]),
            "oracle_pack": (None, [vp, i64, i64, vp]),
            "oracle_unpack": (None, [vp, i64, i64, vp]),
            "oracle_quantize_act": (None, [vp, i64, i64, vp, vp, vp]),
            "oracle_rmsnorm": (None, [vp, i64, i64, vp, f32, vp]),
            "oracle_ternary_acc": (None, [vp, vp, i64, i64, i64, vp]),
            "oracle_rescale": (None, [vp, vp, f32, i64, i64, vp]),
            "oracle_to_bf16": (None, [vp, i64, vp]),
            "oracle_absmax": (f32, [vp, i64]),
            "oracle_binary_signs": (None, [vp, i64, i64, ctypes.c_int, vp]),
            "oracle_binary_acc": (None, [vp, vp, i64, i64, vp]),
            "oracle_binary_rescale": (None, [vp, f32, f32, i64, vp]),
            "oracle_bitplanes": (None, [vp, i64, i64, vp, vp]),
            "oracle_bitplane_acc": (None, [vp, vp, vp, i64, i64, vp]),
            "oracle_rope": (None, [vp, i64, i64, i64, ctypes.c_double, vp]),
            "oracle_attention_decode": (None, [vp, vp, vp, i64, i64, i64, i64, i64, vp]),
            "oracle_relu2_gate": (None, [vp, vp, i64, vp]),
            "oracle_residual_add": (None, [vp, vp, i64, vp]),
            "oracle_num_threads": (ctypes.c_int, []),
            "oracle_set_num_threads": (None, [ctypes.c_int]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# ternary path
# --------------------------------------------------------------------------

def weight_scale(W: np.ndarray) -> np.float32:
    """gamma_eff = max(mean|W| (fp64 sum, row order, rounded to fp32), 1e-5)."""
    W = _c(W, np.float32)
    N, K = W.shape
    return np.float32(_load().oracle_weight_scale(_p(W), N, K))


def ternary_codes(W: np.ndarray, gamma_eff) -> np.ndarray:
    """code = clamp(rint(W / gamma_eff), -1, 1) as int8 [N, K]."""
    W = _c(W, np.float32)
    N, K = W.shape
    out = np.empty((N, K), np.int8)
    _load().oracle_ternary_codes(_p(W), N, K, float(np.float32(gamma_eff)), _p(out))
    return out


def num_threads() -> int:
    """Threads the oracle's parallel loops use."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Thread count for the oracle's parallel loops (timing only; results do not depend on it)."""
    _load().oracle_set_num_threads(int(n))


def packed_bytes(N: int, K: int) -> int:
    return int(_load().oracle_packed_bytes(N, K))


def pack(codes: np.ndarray) -> np.ndarray:
    """Signed codes [N, K] -> TL packed bytes (uint8, flat)."""
    codes = _c(codes, np.int8)
    N, K = codes.shape
    if K % 64:
        raise ValueError("K must be a multiple of 64")
    out = np.empty(packed_bytes(N, K), np.uint8)
    _load().oracle_pack(_p(codes), N, K, _p(out))
    return out


def unpack(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    packed = _c(packed, np.uint8)
    out = np.empty((N, K), np.int8)
    _load().oracle_unpack(_p(packed), N, K, _p(out))
    return out


def quantize_act(x: np.ndarray):
    """Per-token absmax int8: returns (q int8 [M,K], d fp32 [M], rowsum int32 [M])."""
    x = _c(x, np.float32)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    d = np.empty(M, np.float32)
    r = np.empty(M, np.int32)
    _load().oracle_quantize_act(_p(x), M, K, _p(q), _p(d), _p(r))
    return q, d, r


RMS_EPS = 1e-5  # the reading's default epsilon


def rmsnorm(x: np.ndarray, gain=None, eps: float = RMS_EPS) -> np.ndarray:
    """h = (x * r) * gain with r = 1 / sqrt(mean(x^2) + eps): the mean square
    summed in fp64 and rounded once to fp32, everything after it in fp32
    (correctly rounded square root and division).  fp32 [M, K]."""
    x = _c(x, np.float32)
    M, K = x.shape
    h = np.empty((M, K), np.float32)
    g = None if gain is None else _c(np.asarray(gain).reshape(-1), np.float32)
    if g is not None and g.size != K:
        raise ValueError("gain must have K elements")
    _load().oracle_rmsnorm(_p(x), M, K, None if g is None else _p(g),
                           float(np.float32(eps)), _p(h))
    return h


def rmsnorm_quantize_act(x: np.ndarray, gain=None, eps: float = RMS_EPS):
    """RMSNorm, then per-token absmax int8: (q, d, rowsum) of the normalised rows."""
    return quantize_act(rmsnorm(x, gain, eps))


def ternary_acc(codes: np.ndarray, q: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k codes[n, k] * q[m, k] (int32 [M, N])."""
    codes = _c(codes, np.int8)
    q = _c(q, np.int8)
    N, K = codes.shape
    M = q.shape[0]
    assert q.shape[1] == K
    acc = np.empty((M, N), np.int32)
    _load().oracle_ternary_acc(_p(codes), _p(q), M, N, K, _p(acc))
    return acc


def rescale(acc: np.ndarray, d: np.ndarray, gamma_eff) -> np.ndarray:
    acc = _c(acc, np.int32)
    d = _c(d, np.float32)
    M, N = acc.shape
    y = np.empty((M, N), np.float32)
    _load().oracle_rescale(_p(acc), _p(d), float(np.float32(gamma_eff)), M, N, _p(y))
    return y


def to_bf16_bits(y: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even."""
    y = _c(y, np.float32)
    out = np.empty(y.shape, np.uint16)
    _load().oracle_to_bf16(_p(y), y.size, _p(out))
    return out


def bitlinear(x: np.ndarray, W: np.ndarray):
    """The whole ternary path on fp32 inputs; returns a dict of every stage."""
    g = weight_scale(W)
    codes = ternary_codes(W, g)
    q, d, r = quantize_act(x)
    acc = ternary_acc(codes, q)
    y = rescale(acc, d, g)
    return {"gamma": g, "codes": codes, "q": q, "d": d, "rowsum": r,
            "acc": acc, "y": y}


def gemv_from_codes(codes: np.ndarray, gamma_eff, x: np.ndarray):
    """Quantise x, multiply by given codes and rescale (the per-call decode path)."""
    q, d, r = quantize_act(x)
    acc = ternary_acc(codes, q)
    return rescale(acc, d, gamma_eff), acc, q, d, r


# --------------------------------------------------------------------------
# binary path
# --------------------------------------------------------------------------

def absmax(v: np.ndarray) -> np.float32:
    v = _c(v, np.float32)
    return np.float32(_load().oracle_absmax(_p(v), v.size))


def binary_signs(v: np.ndarray, pad_bit: int = 0) -> np.ndarray:
    """Rows of v [R, K] -> uint64 [R, ceil(K/64)], bit = (v < 0)."""
    v = _c(v, np.float32)
    R, K = v.shape
    out = np.empty((R, (K + 63) // 64), np.uint64)
    _load().oracle_binary_signs(_p(v), R, K, int(pad_bit), _p(out))
    return out


def binary_acc(Wb: np.ndarray, xb: np.ndarray, K: int) -> np.ndarray:
    Wb = _c(Wb, np.uint64)
    xb = _c(xb, np.uint64).reshape(-1)
    N = Wb.shape[0]
    acc = np.empty(N, np.int32)
    _load().oracle_binary_acc(_p(Wb), _p(xb), N, K, _p(acc))
    return acc


def binary_rescale(acc: np.ndarray, s_w, s_x) -> np.ndarray:
    acc = _c(acc, np.int32)
    y = np.empty(acc.shape, np.float32)
    _load().oracle_binary_rescale(_p(acc), float(np.float32(s_w)),
                                  float(np.float32(s_x)), acc.size, _p(y))
    return y


def binary_gemv(W: np.ndarray, x: np.ndarray):
    """Binary 1-bit GEMV of one token x [K] against W [N, K]."""
    W = _c(W, np.float32)
    x = _c(x, np.float32).reshape(1, -1)
    K = W.shape[1]
    Wb = binary_signs(W, pad_bit=0)
    xb = binary_signs(x, pad_bit=1)
    s_w = absmax(W)
    s_x = absmax(x)
    acc = binary_acc(Wb, xb, K)
    return {"Wb": Wb, "xb": xb, "s_w": s_w, "s_x": s_x, "acc": acc,
            "y": binary_rescale(acc, s_w, s_x)}


# --------------------------------------------------------------------------
# ternary weights x 1-bit activations (two bit-planes)
# --------------------------------------------------------------------------

def bitplanes(codes: np.ndarray):
    """Signed codes [N, K] -> (mag, sign) uint64 [N, ceil(K/64)]: mag bit set
    for a non-zero weight, sign bit set for a negative one."""
    codes = _c(codes, np.int8)
    N, K = codes.shape
    words = (K + 63) // 64
    mag = np.empty((N, words), np.uint64)
    sign = np.empty((N, words), np.uint64)
    _load().oracle_bitplanes(_p(codes), N, K, _p(mag), _p(sign))
    return mag, sign


def bitplane_acc(mag: np.ndarray, sign: np.ndarray, xb: np.ndarray, K: int) -> np.ndarray:
    """dot[n] = popc(mag & XNOR(sign, x)) - popc(mag & XOR(sign, x)) over the row."""
    mag = _c(mag, np.uint64)
    sign = _c(sign, np.uint64)
    xb = _c(xb, np.uint64).reshape(-1)
    N = mag.shape[0]
    acc = np.empty(N, np.int32)
    _load().oracle_bitplane_acc(_p(mag), _p(sign), _p(xb), N, K, _p(acc))
    return acc


def bitplane_gemv(codes: np.ndarray, gamma_eff, x: np.ndarray):
    """Ternary codes [N, K] against the sign bits of one token x [K]:
    y = (float)dot * (gamma_eff * max|x|)."""
    x = _c(x, np.float32).reshape(1, -1)
    K = codes.shape[1]
    mag, sign = bitplanes(codes)
    xb = binary_signs(x, pad_bit=0)
    s_x = absmax(x)
    acc = bitplane_acc(mag, sign, xb, K)
    return {"mag": mag, "sign": sign, "xb": xb, "s_x": s_x, "acc": acc,
            "y": binary_rescale(acc, gamma_eff, s_x)}


# --------------------------------------------------------------------------
# decoder layer pieces around the BitLinears (synthetic layer stack)
# --------------------------------------------------------------------------

ROPE_BASE = 10000.0


def rope(x: np.ndarray, heads: int, D: int, pos: int, base: float = ROPE_BASE) -> np.ndarray:
    """Rotate pairs (2i, 2i+1) of each head by pos * base^(-2i/D); fp32 [heads*D]."""
    x = _c(x, np.float32).reshape(-1)
    assert x.size == heads * D
    out = np.empty(heads * D, np.float32)
    _load().oracle_rope(_p(x), heads, D, pos, float(base), _p(out))
    return out


def attention_decode(q, K, V, H: int, Hkv: int, D: int, T: int) -> np.ndarray:
    """Softmax attention of one query token over positions 0..T-1 of a
    [Hkv, T_stride, D] cache (grouped heads); fp32 [H*D] before rounding."""
    q = _c(q, np.float32).reshape(-1)
    K = _c(K, np.float32)
    V = _c(V, np.float32)
    T_stride = K.shape[1]
    out = np.empty(H * D, np.float32)
    _load().oracle_attention_decode(_p(q), _p(K), _p(V), H, Hkv, D, T, T_stride, _p(out))
    return out


def relu2_gate(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    g = _c(g, np.float32).reshape(-1)
    u = _c(u, np.float32).reshape(-1)
    out = np.empty(g.size, np.float32)
    _load().oracle_relu2_gate(_p(g), _p(u), g.size, _p(out))
    return out


def residual_add(h: np.ndarray, y: np.ndarray) -> np.ndarray:
    h = _c(h, np.float32).reshape(-1)
    y = _c(y, np.float32).reshape(-1)
    out = np.empty(h.size, np.float32)
    _load().oracle_residual_add(_p(h), _p(y), h.size, _p(out))
    return out


def bf16_round(v: np.ndarray) -> np.ndarray:
    """fp32 values rounded to bf16 (nearest even), returned as fp32."""
    bits = to_bf16_bits(np.asarray(v, np.float32))
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _linear32(x32: np.ndarray, codes: np.ndarray, gamma, gain=None, eps: float = RMS_EPS):
    """One token's BitLinear: optional RMSNorm, absmax int8, ternary product,
    rescale; fp32 y (before any rounding)."""
    x32 = np.asarray(x32, np.float32).reshape(1, -1)
    if gain is not None:
        x32 = rmsnorm(x32, gain, eps)
    q, d, r = quantize_act(x32)
    return rescale(ternary_acc(codes, q), d, gamma)[0]


def decoder_layer(h: np.ndarray, layer: dict, cache_k: np.ndarray, cache_v: np.ndarray,
                  pos: int, cfg: dict) -> np.ndarray:
    """One decode step of one layer (readings as in the C functions above):
    h (bf16 values as fp32 [hidden]) -> new h; writes position pos of the
    layer's cache [Hkv, T, D] (bf16 values as fp32).  layer: dict of
    (gamma, codes) for q, k, v, o, gate, up, down and the two RMSNorm gains
    (fp32 arrays) g_attn, g_ffn."""
    H, Hkv, D = cfg["heads"], cfg["kv_heads"], cfg["head_dim"]
    eps = cfg.get("eps", RMS_EPS)
    base = cfg.get("rope_base", ROPE_BASE)
    h = np.asarray(h, np.float32).reshape(-1)
    q = bf16_round(_linear32(h, layer["q"][1], layer["q"][0], layer["g_attn"], eps))
    k = bf16_round(_linear32(h, layer["k"][1], layer["k"][0], layer["g_attn"], eps))
    v = bf16_round(_linear32(h, layer["v"][1], layer["v"][0], layer["g_attn"], eps))
    q_rot = bf16_round(rope(q, H, D, pos, base))
    k_rot = bf16_round(rope(k, Hkv, D, pos, base))
    cache_k[:, pos, :] = k_rot.reshape(Hkv, D)
    cache_v[:, pos, :] = v.reshape(Hkv, D)
    attn = bf16_round(attention_decode(q_rot, cache_k, cache_v, H, Hkv, D, pos + 1))
    y_o = _linear32(attn, layer["o"][1], layer["o"][0])
    h1 = bf16_round(residual_add(h, y_o))
    gate = bf16_round(_linear32(h1, layer["gate"][1], layer["gate"][0], layer["g_ffn"], eps))
    up = bf16_round(_linear32(h1, layer["up"][1], layer["up"][0], layer["g_ffn"], eps))
    m = relu2_gate(gate, up)
    y_d = _linear32(m, layer["down"][1], layer["down"][0])
    return bf16_round(residual_add(h1, y_d))
