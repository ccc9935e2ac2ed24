"""Shared helpers for the GPU parity tests: seeded inputs, oracle evaluation
and comparisons.  Expected values come only from ``oracle/``."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth_inputs as si

# Stated floating-point bar for rescaled outputs: relative error <= 1e-3
# against the oracle (bf16 and fp32 outputs).  The integer stages (codes,
# packed bytes, q, rowsum, acc) must match bit for bit.
REL_TOL = 1e-3


def dev():
    return torch.device("cuda", 0)


def oracle_weight(W: torch.Tensor):
    """gamma_eff, signed codes and TL bytes of a CPU fp32 weight."""
    Wn = W.float().numpy()
    g = oracle.weight_scale(Wn)
    codes = oracle.ternary_codes(Wn, g)
    return g, codes, oracle.pack(codes)


def f32_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def bf16_bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def assert_rel(got: np.ndarray, want: np.ndarray, rel: float = REL_TOL):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    bound = rel * np.abs(want)
    bad = ~(err <= bound)
    # exact zeros on both sides pass with err == 0 <= 0
    assert not bad.any(), (
        f"{int(bad.sum())} of {bad.size} outside rel {rel}: "
        f"first at {np.argwhere(bad)[0]} got {got[bad][0]} want {want[bad][0]}")


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def compare_outputs(y_gpu: torch.Tensor, y32_oracle: np.ndarray):
    """bf16 or fp32 GPU output against the oracle's fp32 y (rounded like it)."""
    if y_gpu.dtype == torch.bfloat16:
        want_bits = oracle.to_bf16_bits(y32_oracle)
        got_bits = bf16_bits_of(y_gpu)
        assert_rel(bf16_to_f32(got_bits), bf16_to_f32(want_bits))
        np.testing.assert_array_equal(got_bits, want_bits)
    else:
        got = y_gpu.detach().cpu().numpy()
        assert_rel(got, y32_oracle)
        np.testing.assert_array_equal(f32_bits(got), f32_bits(y32_oracle))


class Guarded:
    """A device buffer with canary bytes on both sides of the usable span."""

    GUARD = 4096

    def __init__(self, numel: int, dtype: torch.dtype, device):
        esz = torch.empty((), dtype=dtype).element_size()
        g = self.GUARD // esz
        self.full = torch.empty(numel + 2 * g, dtype=dtype, device=device)
        self.full.view(torch.uint8).fill_(0xA5)
        self.g = g
        self.view = self.full[g:g + numel]

    def intact(self) -> bool:
        b = self.full.view(torch.uint8).cpu().numpy()
        gb = self.GUARD
        return bool((b[:gb] == 0xA5).all() and (b[-gb:] == 0xA5).all())


def seeded_problem(N: int, K: int, M: int, seed: int, xdtype=torch.bfloat16, outliers=True):
    W = si.weight(N, K, seed=seed)
    x = si.activations(M, K, seed=seed, outliers=outliers, dtype=xdtype)
    return W, x
