"""A synthetic BitNet b1.58 decoder-layer stack for decode, on the library's
kernels: every layer is five launches (RMSNorm + q/k/v BitLinears; RoPE +
KV-cache append + attention; o BitLinear + residual; RMSNorm + gate/up
BitLinears; squared-ReLU gate + down BitLinear + residual), chained with
programmatic dependent launch, one position advance per token, and the whole
token capturable in a CUDA graph.

Pages: "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete
Guide", sections "Understanding the Two-Phase Architecture" (Attention and
FeedForward call the BitLinear kernel; a KV cache of shape (1, seq_len,
kv_heads, 1, head_dim)), "Running BitNet Inference with CUDA Acceleration"
and "Key Components and Source Code Architecture" (CUDA graphs remove launch
overhead in decode); "bit-floor" README, section "What's inside" (RMSNorm,
RoPE, attention).  The layer order is the plainest reading: pre-norm
attention and feed-forward blocks with residual adds; the pages name no
feed-forward activation, and the squared-ReLU gate is this library's
reading.  Weights are random (seeded, N(0, 0.02^2) absmean-packed); there
is no tokenizer, embedding or sampling: a decode step maps the residual
stream of one token through the layers.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import (BL_ACT_PLAIN, BL_ACT_RELU2_GATE, BL_ACT_RMSNORM, attention_decode,
               attention_workspace, decode_linear, pack, position_advance, rope_table)


@dataclass
class DecoderConfig:
    hidden: int = 2560
    heads: int = 20
    kv_heads: int = 5
    head_dim: int = 128
    ffn: int = 6912
    layers: int = 30
    max_seq: int = 4096
    eps: float = 1e-5
    rope_base: float = 10000.0


@dataclass
class DecoderLayer:
    q: object
    k: object
    v: object
    o: object
    gate: object
    up: object
    down: object
    g_attn: torch.Tensor
    g_ffn: torch.Tensor
    cache_k: torch.Tensor
    cache_v: torch.Tensor


@dataclass
class Decoder:
    cfg: DecoderConfig
    layers: list
    h: torch.Tensor            # residual stream of the current token, bf16 [hidden]
    pos: torch.Tensor          # int32 [1]: the current token's position
    scratch: dict = field(default_factory=dict)

    @classmethod
    def random(cls, cfg: DecoderConfig, seed: int = 0, device="cuda"):
        gen = torch.Generator(device=device)
        layers = []
        D, Hkv = cfg.head_dim, cfg.kv_heads
        shapes = {"q": (cfg.heads * D, cfg.hidden), "k": (Hkv * D, cfg.hidden),
                  "v": (Hkv * D, cfg.hidden), "o": (cfg.hidden, cfg.heads * D),
                  "gate": (cfg.ffn, cfg.hidden), "up": (cfg.ffn, cfg.hidden),
                  "down": (cfg.hidden, cfg.ffn)}
        for li in range(cfg.layers):
            w = {}
            for j, (name, (N, K)) in enumerate(shapes.items()):
                gen.manual_seed(seed * 1_000_003 + li * 101 + j)
                W = torch.randn(N, K, generator=gen, device=device, dtype=torch.float32) * 0.02
                w[name] = pack(W)
                del W
            gains = []
            for j in range(2):
                gen.manual_seed(seed * 1_000_003 + li * 101 + 50 + j)
                g = 1.0 + 0.1 * torch.randn(cfg.hidden, generator=gen, device=device)
                gains.append(g.to(torch.bfloat16))
            ck = torch.zeros(Hkv, cfg.max_seq, D, dtype=torch.bfloat16, device=device)
            cv = torch.zeros_like(ck)
            layers.append(DecoderLayer(w["q"], w["k"], w["v"], w["o"], w["gate"], w["up"],
                                       w["down"], gains[0], gains[1], ck, cv))
        h = torch.zeros(cfg.hidden, dtype=torch.bfloat16, device=device)
        pos = torch.zeros(1, dtype=torch.int32, device=device)
        dec = cls(cfg, layers, h, pos)
        dec._alloc()
        return dec

    @classmethod
    def from_weights(cls, cfg: DecoderConfig, layers_w: list, device="cuda"):
        """layers_w: per layer a dict of fp32 weights q, k, v, o, gate, up, down
        ([N, K], any device) and gains g_attn, g_ffn ([hidden]); packed here."""
        layers = []
        for w in layers_w:
            pk = {n: pack(w[n].to(device)) for n in ("q", "k", "v", "o", "gate", "up", "down")}
            ck = torch.zeros(cfg.kv_heads, cfg.max_seq, cfg.head_dim, dtype=torch.bfloat16,
                             device=device)
            layers.append(DecoderLayer(pk["q"], pk["k"], pk["v"], pk["o"], pk["gate"], pk["up"],
                                       pk["down"], w["g_attn"].to(device), w["g_ffn"].to(device),
                                       ck, torch.zeros_like(ck)))
        h = torch.zeros(cfg.hidden, dtype=torch.bfloat16, device=device)
        pos = torch.zeros(1, dtype=torch.int32, device=device)
        dec = cls(cfg, layers, h, pos)
        dec._alloc()
        return dec

    def _alloc(self):
        c, dev = self.cfg, self.h.device
        bf = torch.bfloat16
        self.scratch = {"q": torch.empty(c.heads * c.head_dim, dtype=bf, device=dev),
                        "k": torch.empty(c.kv_heads * c.head_dim, dtype=bf, device=dev),
                        "v": torch.empty(c.kv_heads * c.head_dim, dtype=bf, device=dev),
                        "attn": torch.empty(c.heads * c.head_dim, dtype=bf, device=dev),
                        "gate": torch.empty(c.ffn, dtype=bf, device=dev),
                        "up": torch.empty(c.ffn, dtype=bf, device=dev),
                        "attn_ws": attention_workspace(c.heads, c.kv_heads, c.max_seq, dev),
                        "rope": rope_table(c.max_seq, c.rope_base, dev)}

    def set_position(self, pos: int):
        self.pos.fill_(int(pos))

    def layer_step(self, L: DecoderLayer, pdl: bool = True):
        """One layer for the current token (five launches)."""
        c, s, h = self.cfg, self.scratch, self.h
        decode_linear([L.q, L.k, L.v], h, BL_ACT_RMSNORM, gain=L.g_attn, eps=c.eps,
                      outs=[s["q"], s["k"], s["v"]], pdl=pdl)
        attention_decode(s["q"], s["k"], s["v"], L.cache_k, L.cache_v, self.pos, c.heads,
                         c.kv_heads, out=s["attn"], rope_base=c.rope_base,
                         workspace=s["attn_ws"], table=s["rope"], pdl=pdl)
        decode_linear([L.o], s["attn"], BL_ACT_PLAIN, outs=[h], resid=[h], pdl=pdl)
        decode_linear([L.gate, L.up], h, BL_ACT_RMSNORM, gain=L.g_ffn, eps=c.eps,
                      outs=[s["gate"], s["up"]], pdl=pdl)
        decode_linear([L.down], s["gate"], BL_ACT_RELU2_GATE, x2=s["up"], outs=[h], resid=[h],
                      pdl=pdl)

    def step(self, pdl: bool = True):
        """One decode step: the token in self.h through every layer, then the
        position advances.  5 * layers + 1 launches."""
        for L in self.layers:
            self.layer_step(L, pdl)
        position_advance(self.pos)

    def weight_bytes(self) -> int:
        return sum(w.packed.numel() for L in self.layers
                   for w in (L.q, L.k, L.v, L.o, L.gate, L.up, L.down))
