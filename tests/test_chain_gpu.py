"""The persistent decode chain (bitlinear_chain_plan / _run) against the CPU
oracle's chain and against the one-launch-per-step path, through the C ABI.

Each step of a chain reads an earlier step's output, so every step's outputs
are compared with the oracle applied to the oracle's own previous output:
integers bit for bit, outputs bit-identical (within 1e-3 relative a fortiori).
The timeout test makes one bounded wait run out on purpose (an arrival count
nothing reaches) and checks that the launch returns, the status word reads
BL_ERR_TIMEOUT, and the device keeps working.
"""
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


def _bits_to_bf16(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


def _oracle_step(ws_o, x_bf16, gain=None, eps=1e-5):
    """ws_o: list of (gamma, codes); x: bf16 [1, K].  Returns per product
    (y32, acc, bf16 bits)."""
    xf = x_bf16.float().numpy()
    if gain is not None:
        xf = oracle.rmsnorm(xf, gain.float().cpu().numpy(), eps)
    q, d, r = oracle.quantize_act(xf)
    out = []
    for g, codes in ws_o:
        acc = oracle.ternary_acc(codes, q)
        y = oracle.rescale(acc, d, g)
        out.append((y, acc, oracle.to_bf16_bits(y)))
    return out


LAYER = [("qkv", [("q", 2560, 2560), ("k", 2560, 640), ("v", 2560, 640)]),
         ("o", [("o", 2560, 2560)]),
         ("gate_up", [("gate", 2560, 6912), ("up", 2560, 6912)]),
         ("down", [("down", 6912, 2560)])]


def _build_layers(bl, layers, seed, norm=False):
    """Packed weights (GPU) and their oracle codes, outputs, and the chain of
    steps of `layers` decoder layers of 2.4B shapes."""
    x0 = si.activations(1, 2560, seed=seed)
    x0d = x0.to(dev())
    steps, oracle_steps = [], []
    h = x0d
    for layer in range(layers):
        outs_of = {}
        for li, (lname, prods) in enumerate(LAYER):
            ws, ws_o, outs, accs = [], [], [], []
            for j, (name, K, N) in enumerate(prods):
                W = si.weight(N, K, seed=seed * 1000 + layer * 10 + li * 3 + j)
                g, codes, _ = oracle_weight(W)
                ws.append(bl.pack(W.to(dev())))
                ws_o.append((g, codes))
                outs.append(torch.full((1, N), float("nan"), dtype=torch.bfloat16, device=dev()))
                accs.append(torch.zeros(1, N, dtype=torch.int32, device=dev()))
            gain = None
            if norm and lname in ("qkv", "gate_up"):
                gain = (1.0 + 0.2 * si.activations(1, prods[0][1], seed=layer * 7 + li,
                                                   outliers=False, dtype=torch.float32)[0]
                        ).to(torch.bfloat16).to(dev())
            x_in = {"qkv": h, "o": None, "gate_up": None, "down": None}[lname]
            if lname == "o":
                x_in = outs_of["qkv"][0]
            elif lname == "gate_up":
                x_in = outs_of["o"][0]
            elif lname == "down":
                x_in = outs_of["gate_up"][0]
            outs_of[lname] = outs
            steps.append(bl.ChainStep(ws, x_in, outs, gain=gain, acc_dbgs=accs))
            oracle_steps.append((lname, ws_o, gain))
        h = outs_of["down"][0]
    return x0, steps, oracle_steps


def _check_against_oracle(x0, steps, oracle_steps):
    prev = {}
    h = x0
    for st, (lname, ws_o, gain) in zip(steps, oracle_steps):
        x = {"qkv": h, "o": prev.get("qkv"), "gate_up": prev.get("o"),
             "down": prev.get("gate_up")}[lname]
        res = _oracle_step(ws_o, x, gain)
        for (y32, acc, bits), out, a in zip(res, st.outs, st.acc_dbgs):
            np.testing.assert_array_equal(a.cpu().numpy(), acc)
            compare_outputs(out, y32)
        prev[lname] = _bits_to_bf16(res[0][2])
        if lname == "down":
            h = prev["down"]


@pytest.mark.parametrize("layers,norm", [(2, False), (2, True)])
def test_chain_matches_oracle(bl, layers, norm):
    x0, steps, oracle_steps = _build_layers(bl, layers, seed=3 + layers, norm=norm)
    chain = bl.DecodeChain(steps)
    chain.run()
    torch.cuda.synchronize()
    assert bl.last_device_status() == 0
    _check_against_oracle(x0, steps, oracle_steps)


def test_chain_equals_per_launch_path_in_a_graph_and_repeats(bl):
    """Four layers: the chain replayed from a CUDA graph three times gives,
    every time, exactly the outputs of the one-launch-per-step path."""
    x0, steps, _ = _build_layers(bl, 4, seed=11)
    ref = [[torch.empty_like(o) for o in st.outs] for st in steps]
    # the per-launch path reads the chain's own buffers as inputs: run the
    # chain first, then compare step by step on identical inputs
    chain = bl.DecodeChain(steps)
    chain.run()
    torch.cuda.synchronize()
    for st, r in zip(steps, ref):
        bl.gemv_fused_multi(st.weights, st.x, outs=r)
    torch.cuda.synchronize()
    for st, r in zip(steps, ref):
        for o, rr in zip(st.outs, r):
            assert torch.equal(o.view(torch.int16), rr.view(torch.int16))
    snapshot = [[o.clone() for o in st.outs] for st in steps]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        chain.run()
    for _ in range(3):
        for st in steps:
            for o in st.outs:
                o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for st, snap in zip(steps, snapshot):
            for o, s0 in zip(st.outs, snap):
                assert torch.equal(o.view(torch.int16), s0.view(torch.int16))
    assert bl.last_device_status() == 0


def test_chain_sparse_and_mixed_steps(bl):
    """Steps with fewer row groups than CTAs (most CTAs idle in them), fp32
    input and output, K = 8192 and 16384, and a step whose input is the
    output of a step two back."""
    K1, K2 = 8192, 16384
    specs = [(K1, [8]), (K1, [K2]), (K2, [13, 1001]), (K2, [K1])]
    ws_all, oracle_all, steps = [], [], []
    x0 = si.activations(1, K1, seed=21, dtype=torch.float32)
    xs = [x0.to(dev())]
    for i, (K, Ns) in enumerate(specs):
        ws, wo, outs, accs = [], [], [], []
        for j, N in enumerate(Ns):
            W = si.weight(N, K, seed=700 + 10 * i + j)
            g, codes, _ = oracle_weight(W)
            ws.append(bl.pack(W.to(dev())))
            wo.append((g, codes))
            outs.append(torch.full((1, N), float("nan"), dtype=torch.float32, device=dev()))
            accs.append(torch.zeros(1, N, dtype=torch.int32, device=dev()))
        x_in = {0: xs[0], 1: xs[0], 2: None, 3: None}[i]
        if i == 2:
            x_in = steps[1].outs[0]          # K2 outputs of step 1
        if i == 3:
            x_in = steps[1].outs[0]          # two steps back
        steps.append(bl.ChainStep(ws, x_in, outs, acc_dbgs=accs))
        oracle_all.append(wo)
    chain = bl.DecodeChain(steps)
    chain.run()
    torch.cuda.synchronize()
    assert bl.last_device_status() == 0
    for i, (st, wo) in enumerate(zip(steps, oracle_all)):
        xin = st.x.cpu().float().numpy()
        q, d, r = oracle.quantize_act(xin)
        for (g, codes), out, a in zip(wo, st.outs, st.acc_dbgs):
            acc = oracle.ternary_acc(codes, q)
            np.testing.assert_array_equal(a.cpu().numpy(), acc)
            compare_outputs(out, oracle.rescale(acc, d, g))


def test_chain_wait_runs_out_and_device_recovers(bl):
    """A wait that nothing satisfies (the timeout hook, 1 ms): the launch
    returns, the status word reads BL_ERR_TIMEOUT, step 0 is still right, and
    a normal run afterwards is exact with a clean status."""
    x0, steps, oracle_steps = _build_layers(bl, 1, seed=31)
    chain = bl.DecodeChain(steps)
    chain.run_timeout_test(1_000_000)
    torch.cuda.synchronize()
    assert bl.last_device_status() == bl.BL_ERR_TIMEOUT
    assert bl.last_device_status() == 0        # read and cleared
    res = _oracle_step(oracle_steps[0][1], x0)
    for (y32, _, _), out in zip(res, steps[0].outs):
        compare_outputs(out, y32)
    chain.run()
    torch.cuda.synchronize()
    assert bl.last_device_status() == 0
    _check_against_oracle(x0, steps, oracle_steps)
