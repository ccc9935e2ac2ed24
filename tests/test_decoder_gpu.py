"""The decoder-layer stack's kernels on the GPU against the CPU oracle:
decode attention (RoPE, KV-cache append, softmax over the cached
positions), the squared-ReLU-gated and residual BitLinear launches, and
whole layers token after token, eager and replayed from a CUDA graph.

Outputs and cache rows must be bit-identical to the oracle's: every
reduction is defined in fp64 and rounded once, so the two sides differ only
if a value lands within about 1e-15 of an fp32 rounding boundary, which the
seeded cases here do not hit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from parity_helpers import bf16_bits_of, compare_outputs, dev, oracle_weight

pytestmark = pytest.mark.gpu

H, HKV, D = 20, 5, 128


@pytest.fixture(scope="module")
def bl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_ternary_weight_b200 as b
    return b


def _bf16(t):
    return t.to(torch.bfloat16)


def _f32_of_bf16(t):
    return t.float().cpu().numpy()


@pytest.mark.parametrize("pos,T_max", [(0, 64), (1, 64), (7, 64), (100, 1024), (1000, 1024),
                                       (4095, 4096)])
def test_attention_decode_parity(bl, pos, T_max):
    g = torch.Generator().manual_seed(pos + T_max)
    q = _bf16(torch.randn(H * D, generator=g))
    k = _bf16(torch.randn(HKV * D, generator=g))
    v = _bf16(torch.randn(HKV * D, generator=g))
    ck = _bf16(torch.randn(HKV, T_max, D, generator=g))
    cv = _bf16(torch.randn(HKV, T_max, D, generator=g))
    ck_d, cv_d = ck.to(dev()), cv.to(dev())
    posd = torch.tensor([pos], dtype=torch.int32, device=dev())
    out = bl.attention_decode(q.to(dev()), k.to(dev()), v.to(dev()), ck_d, cv_d, posd, H, HKV)
    torch.cuda.synchronize()
    assert bl.last_device_status() == 0
    # oracle
    q_rot = oracle.bf16_round(oracle.rope(_f32_of_bf16(q), H, D, pos))
    k_rot = oracle.bf16_round(oracle.rope(_f32_of_bf16(k), HKV, D, pos))
    K = _f32_of_bf16(ck)
    V = _f32_of_bf16(cv)
    K[:, pos] = k_rot.reshape(HKV, D)
    V[:, pos] = _f32_of_bf16(v).reshape(HKV, D)
    want = oracle.attention_decode(q_rot, K, V, H, HKV, D, pos + 1)
    compare_outputs(out.view(1, -1), want.reshape(1, -1))
    np.testing.assert_array_equal(_f32_of_bf16(ck_d), K)
    np.testing.assert_array_equal(_f32_of_bf16(cv_d), V)


def test_attention_position_outside_cache_writes_nothing(bl):
    T_max = 16
    ck = torch.zeros(HKV, T_max, D, dtype=torch.bfloat16, device=dev())
    cv = torch.zeros_like(ck)
    out = torch.full((H * D,), 3.0, dtype=torch.bfloat16, device=dev())
    x = torch.ones(H * D, dtype=torch.bfloat16, device=dev())
    posd = torch.tensor([T_max], dtype=torch.int32, device=dev())
    bl.attention_decode(x, x[:HKV * D], x[:HKV * D], ck, cv, posd, H, HKV, out=out)
    torch.cuda.synchronize()
    assert bl.last_device_status() == bl.BL_ERR_SHAPE
    assert not ck.any() and not cv.any() and (out == 3.0).all()


@pytest.mark.parametrize("K,N", [(6912, 2560), (2560, 2560), (2304, 1001)])
def test_relu2_gate_and_residual_linear(bl, K, N):
    W = si.weight(N, K, seed=K + N)
    g, codes, _ = oracle_weight(W)
    gate = si.activations(1, K, seed=1, dtype=torch.bfloat16)[0]
    up = si.activations(1, K, seed=2, dtype=torch.bfloat16)[0]
    h = si.activations(1, N, seed=3, dtype=torch.bfloat16)[0]
    w = bl.pack(W.to(dev()))
    hd = h.to(dev())
    acc = torch.empty(N, dtype=torch.int32, device=dev())
    bl.decode_linear([w], gate.to(dev()), bl.BL_ACT_RELU2_GATE, x2=up.to(dev()), outs=[hd],
                     resid=[hd], acc_dbgs=[acc])
    torch.cuda.synchronize()
    m = oracle.relu2_gate(gate.float().numpy(), up.float().numpy())
    q, d, r = oracle.quantize_act(m.reshape(1, -1))
    acc_o = oracle.ternary_acc(codes, q)
    y32 = oracle.rescale(acc_o, d, g)[0]
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o[0])
    want = oracle.residual_add(h.float().numpy(), y32)
    compare_outputs(hd.view(1, -1), want.reshape(1, -1))


def test_plain_linear_with_separate_residual(bl):
    K, N = 2560, 2560
    W = si.weight(N, K, seed=8)
    g, codes, _ = oracle_weight(W)
    x = si.activations(1, K, seed=9)[0]
    h = si.activations(1, N, seed=10)[0]
    w = bl.pack(W.to(dev()))
    y = torch.empty(N, dtype=torch.bfloat16, device=dev())
    bl.decode_linear([w], x.to(dev()), bl.BL_ACT_PLAIN, outs=[y], resid=[h.to(dev())])
    torch.cuda.synchronize()
    q, d, r = oracle.quantize_act(x.float().numpy().reshape(1, -1))
    y32 = oracle.rescale(oracle.ternary_acc(codes, q), d, g)[0]
    compare_outputs(y.view(1, -1), oracle.residual_add(h.float().numpy(), y32).reshape(1, -1))


def _layers_cpu(n_layers, cfg, seed):
    out = []
    for li in range(n_layers):
        shapes = {"q": (cfg.heads * D, cfg.hidden), "k": (cfg.kv_heads * D, cfg.hidden),
                  "v": (cfg.kv_heads * D, cfg.hidden), "o": (cfg.hidden, cfg.heads * D),
                  "gate": (cfg.ffn, cfg.hidden), "up": (cfg.ffn, cfg.hidden),
                  "down": (cfg.hidden, cfg.ffn)}
        w = {n: si.weight(N, K, seed=seed * 100 + li * 10 + j)
             for j, (n, (N, K)) in enumerate(shapes.items())}
        for j, gname in enumerate(("g_attn", "g_ffn")):
            w[gname] = (1.0 + 0.1 * si.activations(1, cfg.hidden, seed=seed * 7 + li * 3 + j,
                                                   outliers=False, dtype=torch.float32)[0]
                        ).to(torch.bfloat16)
        out.append(w)
    return out


def _oracle_layers(layers_w):
    out = []
    for w in layers_w:
        L = {}
        for n in ("q", "k", "v", "o", "gate", "up", "down"):
            g, codes, _ = oracle_weight(w[n])
            L[n] = (g, codes)
        L["g_attn"] = w["g_attn"].float().numpy()
        L["g_ffn"] = w["g_ffn"].float().numpy()
        out.append(L)
    return out


@pytest.mark.parametrize("graph", [False, True])
def test_decoder_stack_tokens_match_oracle(bl, graph):
    """Two layers of 2.4B shapes, a synthetic history of 40 cached positions,
    then four decode tokens: the residual stream after every token and the
    cache rows written must equal the oracle's bit for bit."""
    from bit_ternary_weight_b200.decoder import Decoder, DecoderConfig
    cfg = DecoderConfig(layers=2, max_seq=64)
    layers_w = _layers_cpu(2, cfg, seed=3)
    dec = Decoder.from_weights(cfg, layers_w, device=dev())
    ol = _oracle_layers(layers_w)
    P0 = 40
    cfgd = dict(heads=cfg.heads, kv_heads=cfg.kv_heads, head_dim=D)
    caches = []
    for li, L in enumerate(dec.layers):
        g = torch.Generator().manual_seed(50 + li)
        hist_k = _bf16(torch.randn(cfg.kv_heads, cfg.max_seq, D, generator=g))
        hist_v = _bf16(torch.randn(cfg.kv_heads, cfg.max_seq, D, generator=g))
        hist_k[:, P0:] = 0
        hist_v[:, P0:] = 0
        L.cache_k.copy_(hist_k)
        L.cache_v.copy_(hist_v)
        caches.append((_f32_of_bf16(hist_k), _f32_of_bf16(hist_v)))
    dec.set_position(P0)
    tokens = [si.activations(1, cfg.hidden, seed=200 + t)[0] for t in range(4)]
    if graph:
        dec.h.copy_(tokens[0])
        dec.step()                     # warm-up (token 0, eager)
        torch.cuda.synchronize()
        g_ = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_):
            dec.step()
    for t, tok in enumerate(tokens):
        if not (graph and t == 0):
            dec.h.copy_(tok)
            if graph:
                g_.replay()
            else:
                dec.step()
        torch.cuda.synchronize()
        assert bl.last_device_status() == 0
        h = oracle.bf16_round(tok.float().numpy())
        for L, (ck, cv) in zip(ol, caches):
            h = oracle.decoder_layer(h, L, ck, cv, P0 + t, cfgd)
        np.testing.assert_array_equal(bf16_bits_of(dec.h), oracle.to_bf16_bits(h))
    assert int(dec.pos.item()) == P0 + 4
    for L, (ck, cv) in zip(dec.layers, caches):
        np.testing.assert_array_equal(_f32_of_bf16(L.cache_k), ck)
        np.testing.assert_array_equal(_f32_of_bf16(L.cache_v), cv)


def test_rope_table_and_attention_with_it(bl):
    """The table holds the oracle's cos/sin (fp64, rounded to fp32), and
    attention with the table equals attention without it bit for bit."""
    import math
    T_max = 256
    tab = bl.rope_table(T_max, device=dev()).cpu().numpy()
    for t in (0, 1, 77, 255):
        for i in (0, 1, 31, 63):
            ang = t * 10000.0 ** (-(2.0 * i) / 128)
            assert tab[t, i, 0] == np.float32(math.cos(ang))
            assert tab[t, i, 1] == np.float32(math.sin(ang))
    g = torch.Generator().manual_seed(9)
    q = _bf16(torch.randn(H * D, generator=g)).to(dev())
    k = _bf16(torch.randn(HKV * D, generator=g)).to(dev())
    v = _bf16(torch.randn(HKV * D, generator=g)).to(dev())
    ck = _bf16(torch.randn(HKV, T_max, D, generator=g)).to(dev())
    cv = _bf16(torch.randn(HKV, T_max, D, generator=g)).to(dev())
    posd = torch.tensor([200], dtype=torch.int32, device=dev())
    a = bl.attention_decode(q, k, v, ck.clone(), cv.clone(), posd, H, HKV)
    b = bl.attention_decode(q, k, v, ck.clone(), cv.clone(), posd, H, HKV,
                            table=bl.rope_table(T_max, device=dev()))
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
