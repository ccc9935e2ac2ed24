"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test ties one oracle function to a hand-worked example, a closed form, a
library routine on a special case, a brute-force computation or an invariant,
chosen so that a plausible slip (a dropped term, a wrong sign, a transposed
operand, round-half-away instead of half-even, 128 instead of 127, a per-batch
instead of a per-token scale, a shuffled bit layout) fails at least one test.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si


def _f32(a):
    return np.asarray(a, dtype=np.float32)


# ---------------------------------------------------------------- hand-worked

def test_hand_worked_4x4(golden):
    g = golden("hand_4x4.json")
    W = _f32(g["W"])
    x = _f32(g["x"])
    out = oracle.bitlinear(x, W)
    assert out["gamma"] == pytest.approx(g["gamma"], rel=1e-6)
    np.testing.assert_array_equal(out["codes"], np.array(g["codes"], np.int8))
    np.testing.assert_array_equal(out["q"], np.array(g["q"], np.int8))
    np.testing.assert_array_equal(out["rowsum"], np.array(g["rowsum"], np.int32))
    np.testing.assert_array_equal(out["acc"], np.array(g["acc"], np.int32))
    np.testing.assert_allclose(out["d"], np.array(g["d"]), rtol=1e-6)
    np.testing.assert_allclose(out["y"], np.array(g["y"]), rtol=1e-5, atol=1e-9)


# ---------------------------------------------------------------- rounding ties

def test_code_ties_round_half_even():
    # sum|W| = 4, N*K = 4 -> gamma = 1 exactly; W/gamma = [0.5, -0.5, 1, 2].
    W = _f32([[0.5, -0.5, 1.0, 2.0]])
    g = oracle.weight_scale(W)
    assert g == np.float32(1.0)
    # half-even: 0.5 -> 0, -0.5 -> 0; 2 clips to 1.  Half-away would give +-1.
    np.testing.assert_array_equal(oracle.ternary_codes(W, g), [[0, 0, 1, 1]])


def test_activation_ties_round_half_even():
    # amax = 127 -> s = 1 exactly, so x*s = x.
    x = _f32([[1.5, -1.5, 2.5, -2.5, 0.5, -0.5, 127.0, 0.0]])
    q, d, r = oracle.quantize_act(x)
    np.testing.assert_array_equal(q, [[2, -2, 2, -2, 0, 0, 127, 0]])
    assert d[0] == np.float32(1.0)
    assert r[0] == 127


# ---------------------------------------------------------------- closed forms

def test_weight_scale_closed_forms():
    rng = np.random.default_rng(1)
    # every |w| = 0.25 -> mean |W| = 0.25 exactly whatever the signs
    W = _f32(np.where(rng.random((37, 128)) < 0.5, -0.25, 0.25))
    assert oracle.weight_scale(W) == np.float32(0.25)
    # scaling by a power of two scales gamma exactly and keeps the codes
    W = _f32(rng.standard_normal((64, 192)) * 0.02)
    g = oracle.weight_scale(W)
    assert oracle.weight_scale(W * 4) == g * 4
    np.testing.assert_array_equal(oracle.ternary_codes(W, g),
                                  oracle.ternary_codes(W * 4, g * 4))
    # all-zero weights: gamma clamps to 1e-5 and every code is 0
    Z = np.zeros((8, 64), np.float32)
    assert oracle.weight_scale(Z) == np.float32(1e-5)
    assert not oracle.ternary_codes(Z, oracle.weight_scale(Z)).any()
    # mean|W| of a large Gaussian sample is sigma * sqrt(2/pi)
    W = si.weight(1024, 1024, seed=3).numpy()
    sigma = 0.02
    expect = sigma * math.sqrt(2 / math.pi)
    # std of the mean of |z| over n draws: sigma*sqrt(1-2/pi)/sqrt(n)
    tol = 6 * sigma * math.sqrt(1 - 2 / math.pi) / 1024
    assert abs(float(oracle.weight_scale(W)) - expect) < tol
    # fp64 sum: mean of values that fp32 cannot accumulate exactly
    W = np.full((4096, 4096), np.float32(0.1), np.float32)
    W[0, 0] = np.float32(1e4)
    S = 4096 * 4096 * 0.1 + 1e4 - 0.1
    expect = np.float32(S / (4096 * 4096))
    assert abs(float(oracle.weight_scale(W)) - float(expect)) <= float(np.spacing(expect))


def test_gaussian_zero_fraction():
    # code 0 iff |w| < gamma/2 = sigma*sqrt(2/pi)/2 -> P = erf(sqrt(2/pi)/(2*sqrt(2)))
    W = si.weight(1024, 1024, seed=5).numpy()
    codes = oracle.ternary_codes(W, oracle.weight_scale(W))
    p = math.erf(math.sqrt(2 / math.pi) / (2 * math.sqrt(2)))
    assert abs(p - 0.3101) < 1e-4
    frac = float((codes == 0).mean())
    sd = math.sqrt(p * (1 - p) / codes.size)
    assert abs(frac - p) < 5 * sd
    # the +1 and -1 codes are equally likely by symmetry
    pos, neg = (codes == 1).mean(), (codes == -1).mean()
    assert abs(pos - neg) < 5 * math.sqrt(0.35 * 0.65 / codes.size) * 2


# ---------------------------------------------------------------- quantiser bounds

@pytest.mark.parametrize("M,K", [(1, 64), (3, 256), (16, 2560)])
def test_activation_quant_properties(M, K):
    x = si.activations(M, K, seed=7, dtype=torch.float32).numpy()
    q, d, r = oracle.quantize_act(x)
    amax = np.abs(x).max(axis=1)
    # scale: d = amax / 127 per token (not per batch, not /128)
    np.testing.assert_allclose(d, amax / 127.0, rtol=2e-7)
    # the largest |x| of each token lands on +-127; all |q| <= 127
    assert np.abs(q).max() <= 127
    for m in range(M):
        i = np.argmax(np.abs(x[m]))
        assert abs(int(q[m, i])) == 127
    # round-to-nearest error bound: |x - q*d| <= d/2 (plus fp32 slack)
    err = np.abs(x - q.astype(np.float64) * d[:, None].astype(np.float64))
    assert (err <= d[:, None] * (0.5 + 1e-5)).all()
    # monotone in x within a token
    for m in range(M):
        o = np.argsort(x[m], kind="stable")
        assert (np.diff(q[m, o].astype(np.int32)) >= 0).all()
    # row sums
    np.testing.assert_array_equal(r, q.astype(np.int64).sum(axis=1))
    # scaling a token by a power of two keeps q and scales d exactly
    q2, d2, r2 = oracle.quantize_act(x * 2)
    np.testing.assert_array_equal(q2, q)
    np.testing.assert_array_equal(d2, d * 2)


def test_zero_token():
    x = np.zeros((2, 128), np.float32)
    x[1, 5] = -3.0
    q, d, r = oracle.quantize_act(x)
    assert not q[0].any() and r[0] == 0
    assert d[0] == np.float32(np.float32(1e-5) / np.float32(127.0))
    assert q[1, 5] == -127 and r[1] == -127


def test_codes_round_clip_bound():
    W = si.weight(64, 256, seed=11).numpy()
    g = oracle.weight_scale(W)
    c = oracle.ternary_codes(W, g)
    assert set(np.unique(c)).issubset({-1, 0, 1})
    r = W.astype(np.float64) / float(g)
    inner = np.abs(r) < 1.4999
    # inside the clip range the code is the nearest integer
    assert (np.abs(r[inner] - c[inner]) <= 0.5 + 1e-6).all()
    # outside it the code carries the sign
    outer = np.abs(r) > 1.5001
    assert (c[outer] == np.sign(r[outer])).all()


# ---------------------------------------------------------------- product + rescale

@pytest.mark.parametrize("seed", range(6))
def test_bruteforce_fp64_matmul(seed):
    rng = np.random.default_rng(100 + seed)
    M = int(rng.integers(1, 17))
    N = int(rng.integers(1, 33))
    K = 64 * int(rng.integers(1, 4))
    W = si.weight(N, K, seed=seed).numpy()
    x = si.activations(M, K, seed=seed, dtype=torch.float32).numpy()
    out = oracle.bitlinear(x, W)
    # dequantised operands multiplied in fp64 by numpy (the closed form
    # y = (q d) (codes gamma)^T), against the oracle's integer-then-scale path
    Xd = out["q"].astype(np.float64) * out["d"].astype(np.float64)[:, None]
    Wd = out["codes"].astype(np.float64) * float(out["gamma"])
    ref = Xd @ Wd.T
    np.testing.assert_array_equal(
        out["acc"], (out["q"].astype(np.int64) @ out["codes"].astype(np.int64).T))
    y = out["y"].astype(np.float64)
    tol = 2.5e-7 * np.abs(ref) + 1e-30
    assert (np.abs(y - ref) <= tol).all()


def test_rowsum_identity_and_bounds():
    W = si.weight(40, 512, seed=2).numpy()
    x = si.activations(5, 512, seed=2, dtype=torch.float32).numpy()
    out = oracle.bitlinear(x, W)
    stored = out["codes"].astype(np.int64) + 1
    lhs = out["q"].astype(np.int64) @ stored.T - out["rowsum"][:, None]
    np.testing.assert_array_equal(lhs, out["acc"])
    assert np.abs(out["acc"]).max() <= 127 * 512


def test_permutation_invariance():
    rng = np.random.default_rng(9)
    W = si.weight(16, 320, seed=4).numpy()
    x = si.activations(3, 320, seed=4, dtype=torch.float32).numpy()
    p = rng.permutation(320)
    a = oracle.bitlinear(x, W)
    b = oracle.bitlinear(x[:, p], W[:, p])
    np.testing.assert_array_equal(a["acc"], b["acc"])
    np.testing.assert_array_equal(a["y"], b["y"])


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(3)
    v = rng.standard_normal(4096).astype(np.float32) * 10
    # exact ties between two bf16 values, both parities of the kept bit
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x40498000],
                    np.uint32).view(np.float32)
    v = np.concatenate([v, ties, np.float32([0.0, -0.0, 1e-40, 3.4e38])])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.to_bf16_bits(v), ref)


# ---------------------------------------------------------------- packed layout

def _codes_from_rule(case):
    N, K = case["N"], case["K"]
    c = np.zeros((N, K), np.int8)
    for row, ks, val in case["set"]:
        if ks == "all":
            c[row, :] = val
        else:
            c[row, ks] = val
    return c


def test_layout_hand_fixtures(golden):
    g = golden("tl_layout.json")
    for case in g["cases"]:
        codes = _codes_from_rule(case)
        packed = oracle.pack(codes)
        assert packed.size == case["total_bytes"]
        expect = np.full(case["total_bytes"], case["fill"], np.uint8)
        for off, val in case["bytes"].items():
            expect[int(off)] = val
        np.testing.assert_array_equal(packed, expect)
        np.testing.assert_array_equal(oracle.unpack(packed, case["N"], case["K"]), codes)


@pytest.mark.parametrize("N,K", [(1, 64), (8, 128), (13, 256), (40, 2560)])
def test_pack_roundtrip_and_padding(N, K):
    rng = np.random.default_rng(N * 1000 + K)
    codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    packed = oracle.pack(codes)
    assert packed.size == ((N + 7) // 8) * 8 * K // 4
    np.testing.assert_array_equal(oracle.unpack(packed, N, K), codes)
    # no byte holds the unused value 3 in any 2-bit field
    fields = np.stack([(packed >> s) & 3 for s in (0, 2, 4, 6)])
    assert (fields != 3).all()


def test_packed_words_are_dp4a_ready():
    # (word >> 2i) & 0x03030303 yields the stored codes of four consecutive k
    rng = np.random.default_rng(21)
    N, K = 16, 256
    codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    words = oracle.pack(codes).view("<u4")
    for n in (0, 5, 8, 15):
        for k0 in range(0, K, 16):
            g, r, c, w = n // 8, n % 8, k0 // 64, (k0 % 64) // 16
            word = int(words[((g * (K // 64) + c) * 8 + r) * 4 + w])
            for i in range(4):
                v = (word >> (2 * i)) & 0x03030303
                got = [(v >> (8 * j)) & 0xFF for j in range(4)]
                want = [int(codes[n, k0 + 4 * i + j]) + 1 for j in range(4)]
                assert got == want


# ---------------------------------------------------------------- binary variant

@pytest.mark.parametrize("N,K", [(1, 64), (7, 100), (33, 512), (64, 8192)])
def test_xnor_popcount_identity(N, K):
    W = si.weight(N, K, seed=N + K).numpy()
    x = si.activations(1, K, seed=N + K, dtype=torch.float32).numpy()
    W[0, 0] = -0.0  # sign bit set, but not < 0: counts as +1
    out = oracle.binary_gemv(W, x)
    sw = np.where(W < 0, -1, 1).astype(np.int64)
    sx = np.where(x[0] < 0, -1, 1).astype(np.int64)
    np.testing.assert_array_equal(out["acc"], sw @ sx)
    assert out["s_w"] == np.abs(W).max() and out["s_x"] == np.abs(x).max()
    ref = (sw @ sx).astype(np.float64) * float(out["s_w"]) * float(out["s_x"])
    assert (np.abs(out["y"] - ref) <= 2.5e-7 * np.abs(ref) + 1e-30).all()


def test_binary_bit_order():
    # bit j of word w <-> k = 64 w + j, bit set for negative values
    v = np.ones((1, 128), np.float32)
    v[0, 3] = -1
    v[0, 64 + 60] = -2
    b = oracle.binary_signs(v)
    assert b.shape == (1, 2)
    assert int(b[0, 0]) == 1 << 3 and int(b[0, 1]) == 1 << 60


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_hand_worked(golden):
    g = golden("rmsnorm_hand.json")
    x = _f32(g["x"])
    h = oracle.rmsnorm(x, eps=g["eps"])
    np.testing.assert_array_equal(h, _f32(g["h_no_gain"]))
    h = oracle.rmsnorm(x, gain=_f32(g["gain"]), eps=g["eps"])
    np.testing.assert_array_equal(h, _f32(g["h_gain"]))


@pytest.mark.parametrize("c", [1.0, -2.0, 0.25, 64.0, -1024.0])
def test_rmsnorm_constant_row_gives_the_gain(c):
    # x = c everywhere: mean square c^2, root |c| (exact for powers of two),
    # r = 1/|c| exact, so h = sign(c) * gain exactly when eps = 0
    K = 64
    gain = np.linspace(-3.0, 3.0, K, dtype=np.float32)
    h = oracle.rmsnorm(np.full((1, K), c, np.float32), gain=gain, eps=0.0)
    np.testing.assert_array_equal(h[0], np.sign(c) * gain)


def test_rmsnorm_then_quantise_gives_the_gain_on_a_constant_token():
    """RMSNorm of a constant token is the gain times one common factor, and the
    absmax quantiser removes that factor: with integer gains 1 .. 127 the codes
    are the gains themselves (every x*s lies within a few ulp of an integer,
    far from a rounding tie), d = max h / 127, and the row sum is the sum of
    the gains.  Quantising the raw token instead would give 127 everywhere."""
    K = 254
    gain = (np.arange(K) % 127 + 1).astype(np.float32)
    for c in (1.0, -3.5, 0.01):
        x = np.full((1, K), c, np.float32)
        q, d, r = oracle.rmsnorm_quantize_act(x, gain)
        want = np.sign(c) * gain
        np.testing.assert_array_equal(q[0], want.astype(np.int8))
        assert r[0] == int(want.sum())
        h = oracle.rmsnorm(x, gain)
        assert d[0] == np.float32(np.abs(h).max() / np.float32(127.0))


def test_rmsnorm_power_of_two_scale_invariance():
    x = si.activations(3, 512, seed=4, dtype=torch.float32).numpy()
    gain = 1.0 + 0.1 * si.activations(1, 512, seed=5, outliers=False, dtype=torch.float32).numpy()
    h = oracle.rmsnorm(x, gain=gain, eps=0.0)
    for a in (2.0, 0.125, -8.0):
        np.testing.assert_array_equal(oracle.rmsnorm(x * np.float32(a), gain=gain, eps=0.0),
                                      np.sign(a) * h)


@pytest.mark.parametrize("eps", [0.0, 1e-5, 1e-2])
@pytest.mark.parametrize("scale", [1.0, 1e-3])
def test_rmsnorm_against_fp64_definition(eps, scale):
    # textbook RMSNorm in fp64 (numpy); the fp32 chain (mean rounded to fp32,
    # eps added in fp32, sqrt, divide, two products) stays within a few ulp
    M, K = 4, 2560
    x = (si.activations(M, K, seed=7, dtype=torch.float32).numpy() * np.float32(scale))
    gain = 1.0 + 0.2 * si.activations(1, K, seed=8, outliers=False, dtype=torch.float32).numpy()[0]
    h = oracle.rmsnorm(x, gain=gain, eps=eps).astype(np.float64)
    x64 = x.astype(np.float64)
    ms = (x64 * x64).mean(axis=1, keepdims=True)
    want = x64 / np.sqrt(ms + eps) * gain.astype(np.float64)
    ulp = np.spacing(np.abs(want).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(h - want) <= 4 * ulp + 1e-30)


def test_rmsnorm_eps_dominates_a_tiny_row():
    # mean square 1e-8 << eps = 1e-5: h = x / sqrt(1.001e-5), about 0.0316,
    # not 1 (as it would be without eps)
    x = np.full((1, 256), 1e-4, np.float32)
    h = oracle.rmsnorm(x, eps=1e-5)
    assert h[0, 0] == pytest.approx(1e-4 / math.sqrt(1e-8 + 1e-5), rel=1e-6)


def test_rmsnorm_zero_row_and_quantiser():
    x = np.zeros((2, 128), np.float32)
    x[1, 5] = 3.0
    h = oracle.rmsnorm(x)
    assert not h[0].any()
    q, d, r = oracle.rmsnorm_quantize_act(x)
    assert not q[0].any() and r[0] == 0
    # a one-hot row normalises to 3 / sqrt(9/K + eps) (sqrt(K) without eps) at
    # its position, which quantises to 127
    assert h[1, 5] == pytest.approx(3.0 / math.sqrt(9.0 / 128 + 1e-5), rel=1e-6)
    assert q[1, 5] == 127 and r[1] == 127


# ---------------------------------------------------------------- ternary x 1-bit bit-planes

def test_bitplane_hand_worked():
    # codes [1, 0, -1, 1], x = [2, -3, -1, 0]: mag bits k0, k2, k3 = 0b1101,
    # sign bit k2 = 0b0100, x sign bits k1, k2 = 0b0110.  By hand:
    # sum code * sign(x) = (+1)(+1) + 0 + (-1)(-1) + (+1)(+1) = 3 (x = 0 counts +1)
    codes = np.array([[1, 0, -1, 1]], np.int8)
    mag, sign = oracle.bitplanes(codes)
    assert int(mag[0, 0]) == 0b1101 and int(sign[0, 0]) == 0b0100
    out = oracle.bitplane_gemv(codes, np.float32(0.5), _f32([2.0, -3.0, -1.0, 0.0]))
    assert int(out["xb"][0, 0]) == 0b0110
    assert out["acc"][0] == 3
    assert out["s_x"] == np.float32(3.0)
    assert out["y"][0] == np.float32(3 * 0.5 * 3.0)


@pytest.mark.parametrize("N,K", [(7, 64), (5, 200), (3, 1), (9, 4096)])
def test_bitplane_dot_is_the_signed_product(N, K):
    # brute force: sum_k code[n][k] * (x[k] < 0 ? -1 : +1), zeros and -0.0 included
    rng = np.random.default_rng(N * 1000 + K)
    codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    x = rng.standard_normal(K).astype(np.float32)
    x[rng.integers(0, K, max(1, K // 10))] = 0.0
    x[rng.integers(0, K, max(1, K // 10))] = -0.0
    out = oracle.bitplane_gemv(codes, np.float32(1.0), x)
    sx = np.where(x < 0, -1, 1).astype(np.int64)
    want = (codes.astype(np.int64) * sx[None, :]).sum(axis=1)
    np.testing.assert_array_equal(out["acc"], want)


def test_bitplane_invariants():
    W = si.weight(64, 640, seed=3).numpy()
    g = oracle.weight_scale(W)
    codes = oracle.ternary_codes(W, g)
    mag, sign = oracle.bitplanes(codes)
    # sign bits only where the weight is non-zero; popcount(mag) = non-zeros
    assert not np.any(sign & ~mag)
    nz = np.array([sum(bin(int(v)).count("1") for v in row) for row in mag])
    np.testing.assert_array_equal(nz, (codes != 0).sum(axis=1))
    x = si.activations(1, 640, seed=4, dtype=torch.float32).numpy()[0]
    acc = oracle.bitplane_gemv(codes, g, x)["acc"]
    # |dot| <= non-zeros and dot has their parity
    assert np.all(np.abs(acc) <= nz) and np.all((acc - nz) % 2 == 0)
    # flipping every activation's sign negates every dot product (no x is 0)
    assert np.all(x != 0)
    np.testing.assert_array_equal(oracle.bitplane_gemv(codes, g, -x)["acc"], -acc)


# ---------------------------------------------------------------- decoder layer pieces

def test_rope_hand_and_closed_forms():
    # D = 4: pair 0 turns by pos, pair 1 by pos * 10000^(-1/2) = pos / 100
    out = oracle.rope(_f32([1.0, 0.0, 0.0, 1.0]), 1, 4, 1)
    np.testing.assert_allclose(out, [math.cos(1.0), math.sin(1.0), -math.sin(0.01), math.cos(0.01)],
                               rtol=1e-6, atol=1e-7)
    x = si.activations(1, 8 * 128, seed=2, dtype=torch.float32).numpy()[0]
    np.testing.assert_array_equal(oracle.rope(x, 8, 128, 0), x)       # position 0: identity
    for pos in (1, 17, 1000):
        y = oracle.rope(x, 8, 128, pos).astype(np.float64)
        n_in = x.astype(np.float64).reshape(-1, 2)
        n_out = y.reshape(-1, 2)
        np.testing.assert_allclose(np.hypot(n_out[:, 0], n_out[:, 1]),
                                   np.hypot(n_in[:, 0], n_in[:, 1]), rtol=2e-6, atol=1e-6)
        # against the rotation written in fp64
        i = np.arange(64)
        ang = pos * 10000.0 ** (-(2.0 * i) / 128)
        a, b = n_in[:, 0].reshape(8, 64), n_in[:, 1].reshape(8, 64)
        want = np.stack([a * np.cos(ang) - b * np.sin(ang), a * np.sin(ang) + b * np.cos(ang)], -1)
        np.testing.assert_allclose(y.reshape(8, 64, 2), want, rtol=1e-5, atol=2e-6)


def test_rope_composes():
    x = si.activations(1, 4 * 128, seed=3, dtype=torch.float32).numpy()[0]
    two = oracle.rope(oracle.rope(x, 4, 128, 5), 4, 128, 7)
    np.testing.assert_allclose(two, oracle.rope(x, 4, 128, 12), rtol=1e-5, atol=2e-6)


def test_attention_closed_forms_and_textbook():
    H, Hkv, D, T = 8, 2, 128, 37
    rng = np.random.default_rng(5)
    q = rng.standard_normal(H * D).astype(np.float32)
    K = rng.standard_normal((Hkv, 64, D)).astype(np.float32)
    V = rng.standard_normal((Hkv, 64, D)).astype(np.float32)
    # one position: the softmax is 1, the output is that value row exactly
    out1 = oracle.attention_decode(q, K, V, H, Hkv, D, 1).reshape(H, D)
    for h in range(H):
        np.testing.assert_array_equal(out1[h], V[h // (H // Hkv), 0])
    # textbook softmax attention in fp64 with grouped heads and 1/sqrt(D)
    out = oracle.attention_decode(q, K, V, H, Hkv, D, T).reshape(H, D).astype(np.float64)
    for h in range(H):
        kv = h // (H // Hkv)
        s = (K[kv, :T].astype(np.float64) @ q[h * D:(h + 1) * D]) / math.sqrt(D)
        p = np.exp(s - s.max())
        p /= p.sum()
        np.testing.assert_allclose(out[h], p @ V[kv, :T], rtol=1e-5, atol=1e-6)
    # equal scores (zero query): the mean of the cached values
    out0 = oracle.attention_decode(np.zeros(H * D, np.float32), K, V, H, Hkv, D, T).reshape(H, D)
    np.testing.assert_allclose(out0[0], V[0, :T].mean(axis=0), rtol=1e-5, atol=1e-6)


def test_relu2_gate_and_residual():
    np.testing.assert_array_equal(oracle.relu2_gate(_f32([-1.0, 0.0, 2.0, 0.5]), _f32([3.0, 3.0, 3.0, -4.0])),
                                  _f32([0.0, 0.0, 12.0, -1.0]))
    np.testing.assert_array_equal(oracle.residual_add(_f32([1.0, -2.0]), _f32([0.5, 2.0])), _f32([1.5, 0.0]))


def _layer(seed, zero=(), K=256, H=2, Hkv=1, D=128, F=384):
    hidden = H * D
    shapes = {"q": (hidden, hidden), "k": (Hkv * D, hidden), "v": (Hkv * D, hidden),
              "o": (hidden, hidden), "gate": (F, hidden), "up": (F, hidden), "down": (hidden, F)}
    layer = {}
    for i, (name, (N, Kk)) in enumerate(shapes.items()):
        W = si.weight(N, Kk, seed=seed * 10 + i).numpy()
        if name in zero:
            W = np.zeros_like(W)
        g = oracle.weight_scale(W)
        layer[name] = (g, oracle.ternary_codes(W, g))
    layer["g_attn"] = np.ones(hidden, np.float32)
    layer["g_ffn"] = np.ones(hidden, np.float32)
    return layer, dict(heads=H, kv_heads=Hkv, head_dim=D)


def test_decoder_layer_closed_forms():
    layer, cfg = _layer(1, zero=("q", "k", "v", "o", "gate", "up", "down"))
    h = oracle.bf16_round(si.activations(1, 256, seed=4, dtype=torch.float32).numpy()[0])
    ck = np.zeros((1, 8, 128), np.float32)
    cv = np.zeros((1, 8, 128), np.float32)
    # all weights zero: every BitLinear gives 0, the residual stream is unchanged
    np.testing.assert_array_equal(oracle.decoder_layer(h, layer, ck, cv, 3, cfg), h)
    assert not ck.any() and not cv.any()
    # only the attention output projection and the FFN zero: h is unchanged,
    # and position 3 (only) of the cache is written
    layer, cfg = _layer(2, zero=("o", "gate", "up", "down"))
    ck[:] = 7.0
    out = oracle.decoder_layer(h, layer, ck, cv, 3, cfg)
    np.testing.assert_array_equal(out, h)
    assert (ck[:, [0, 1, 2, 4, 5, 6, 7]] == 7.0).all() and not (ck[:, 3] == 7.0).all()


def _run_layer(layer, cfg, h, pos, T=8):
    ck = np.zeros((cfg["kv_heads"], T, cfg["head_dim"]), np.float32)
    cv = np.zeros_like(ck)
    return oracle.decoder_layer(h, layer, ck, cv, pos, cfg), ck, cv


def _h(seed, positive=False):
    a = si.activations(1, 256, seed=seed, dtype=torch.float32).numpy()[0]
    return oracle.bf16_round(np.abs(a) + 0.25 if positive else a)


def test_decoder_layer_first_position_attends_to_itself():
    """At position 0 the softmax runs over the token's own key: the layer's
    output is finite and differs from its input, and cache row 0 holds the
    token's key and value."""
    layer, cfg = _layer(3)
    h = _h(5)
    out, ck, cv = _run_layer(layer, cfg, h, 0)
    assert np.isfinite(out).all()
    assert (out != h).any()
    assert ck[:, 0].any() and cv[:, 0].any() and not ck[:, 1:].any() and not cv[:, 1:].any()


def test_decoder_layer_each_gain_belongs_to_its_sublayer():
    """A zero RMSNorm gain zeroes every BitLinear input behind it.  Zero
    attention gain and zero FFN weights: the token's q, k, v are 0 (cache row
    0), attention over zero caches gives 0, and the stream is unchanged.  Zero
    FFN gain and zero attention weights: gate = up = 0, unchanged again.  In
    each case the other gain is 1 and the other sublayer's weights are not
    zero, so a gain applied in front of the wrong sublayer shows."""
    layer, cfg = _layer(4, zero=("gate", "up", "down"))
    layer["g_attn"] = np.zeros(256, np.float32)
    h = _h(6)
    out, ck, cv = _run_layer(layer, cfg, h, 2)
    np.testing.assert_array_equal(out, h)
    assert not ck.any() and not cv.any()
    layer, cfg = _layer(5, zero=("q", "k", "v", "o"))
    layer["g_ffn"] = np.zeros(256, np.float32)
    out, _, _ = _run_layer(layer, cfg, h, 2)
    np.testing.assert_array_equal(out, h)


def test_decoder_layer_ffn_adds_to_the_attention_output():
    """Zero FFN weights: the output is the stream after the attention
    residual, which moved (the o projection is not zero)."""
    layer, cfg = _layer(6, zero=("gate", "up", "down"))
    h = _h(7)
    out, _, _ = _run_layer(layer, cfg, h, 1)
    assert (out != h).any()
    # and the FFN with zero weights adds exactly nothing to it: one more
    # layer whose attention is silenced (zero gain) leaves it unchanged
    layer["g_attn"] = np.zeros(256, np.float32)
    out2, _, _ = _run_layer(layer, cfg, out, 1)
    np.testing.assert_array_equal(out2, out)


def test_decoder_layer_gate_is_the_relu_squared_factor():
    """A positive token (after RMSNorm with a positive gain it quantises to
    q >= 0) against gate weights <= 0 gives gate <= 0, so relu(gate)^2 = 0
    closes the FFN whatever up is: with the o projection zero the stream is
    unchanged.  With gate and up exchanged the FFN would not be closed."""
    layer, cfg = _layer(8, zero=("o",))
    Wg = -np.abs(si.weight(384, 256, seed=81).numpy())
    g = oracle.weight_scale(Wg)
    layer["gate"] = (g, oracle.ternary_codes(Wg, g))
    assert (layer["gate"][1] <= 0).all() and (layer["gate"][1] < 0).any()
    h = _h(9, positive=True)
    out, _, _ = _run_layer(layer, cfg, h, 3)
    np.testing.assert_array_equal(out, h)
    # the same layer with gate weights >= 0 does move the stream
    layer["gate"] = (g, -layer["gate"][1])
    out, _, _ = _run_layer(layer, cfg, h, 3)
    assert (out != h).any()


def test_decoder_layer_caches_rotated_keys_and_plain_values():
    """The cached key at position p is the position-0 key (RoPE at 0 is the
    identity) rotated by p; the cached value does not depend on p; a zero
    value projection caches zero values but non-zero keys, and the reverse."""
    layer, cfg = _layer(10)
    h = _h(11)
    _, ck0, cv0 = _run_layer(layer, cfg, h, 0)
    for p in (1, 5):
        _, ckp, cvp = _run_layer(layer, cfg, h, p)
        rot = oracle.bf16_round(oracle.rope(ck0[:, 0].reshape(-1), cfg["kv_heads"],
                                            cfg["head_dim"], p))
        np.testing.assert_array_equal(ckp[:, p].reshape(-1), rot)
        np.testing.assert_array_equal(cvp[:, p], cv0[:, 0])
        assert (ckp[:, p] != ck0[:, 0]).any()
    layer, cfg = _layer(12, zero=("v",))
    _, ck, cv = _run_layer(layer, cfg, h, 2)
    assert ck[:, 2].any() and not cv.any()
    layer, cfg = _layer(13, zero=("k",))
    _, ck, cv = _run_layer(layer, cfg, h, 2)
    assert not ck.any() and cv[:, 2].any()
