"""Column-parallel (N-split) decode: the partition, the packed byte ranges and
the all-gather, on the host.

The split is exact by construction (no partial sum crosses ranks): these
tests check that the rank shards tile the rows and the TL packed bytes, that
each shard's bytes hold exactly its rows' codes, and, with two and three gloo
ranks, that the per-rank oracle outputs gathered through
ColumnParallelDecode equal the unsplit oracle output bit for bit.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth_inputs as si
from bit_ternary_weight_b200.sharding import (ColumnParallelDecode, packed_byte_range,
                                              row_partition, shard_weight)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("N", [1, 7, 8, 9, 640, 1001, 2560, 6912, 28672])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shards_tile_rows_and_packed_bytes(N, world):
    K = 256
    shards = row_partition(N, world)
    assert len(shards) == world
    assert shards[0].row0 == 0 and shards[-1].row1 == N
    R = shards[0].rows_per_rank
    assert R % 8 == 0 and R * world >= N and R * (world - 1) < N + 8 * world
    for a, b in zip(shards, shards[1:]):
        assert a.row1 == b.row0
    # only trailing ranks are short; a short rank is followed by empty ones
    seen_short = False
    for s in shards:
        assert s.rows in range(0, R + 1)
        if seen_short:
            assert s.rows == 0
        seen_short = seen_short or s.rows < R
    ranges = [packed_byte_range(K, s) for s in shards if s.rows]
    assert ranges[0][0] == 0 and ranges[-1][1] == oracle.packed_bytes(N, K)
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0 and a0 < a1
    for b0, _ in ranges:
        assert b0 % 16 == 0   # the GEMV needs 16-byte aligned packed weights


@pytest.mark.parametrize("N,K,world", [(1001, 192, 4), (640, 256, 3), (77, 64, 2)])
def test_shard_bytes_hold_exactly_their_rows(N, K, world):
    W = si.weight(N, K, seed=N + world).numpy()
    g = oracle.weight_scale(W)
    codes = oracle.ternary_codes(W, g)
    packed = oracle.pack(codes)
    from bit_ternary_weight_b200 import TernaryWeight
    w = TernaryWeight(torch.from_numpy(packed), torch.tensor([g]), N, K)
    for s in row_partition(N, world):
        sw = shard_weight(w, s)
        if s.rows == 0:
            assert sw is None
            continue
        assert sw.N == s.rows and sw.K == K and sw.w_scale is w.w_scale
        got = oracle.unpack(sw.packed.numpy(), s.rows, K)
        np.testing.assert_array_equal(got, codes[s.row0:s.row1])


def _free_port() -> int:
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _oracle_y_bits(codes, g, x):
    q, d, r = oracle.quantize_act(x)
    return oracle.to_bf16_bits(oracle.rescale(oracle.ternary_acc(codes, q), d, g))


def _worker(rank, world, port, out_dir, shapes, M):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from bit_ternary_weight_b200 import TernaryWeight
        K = shapes[0][0]
        x = si.activations(M, K, seed=123).float().numpy()
        products, codes_all, gammas = [], [], []
        for i, (_, N) in enumerate(shapes):
            W = si.weight(N, K, seed=300 + i).numpy()
            g = oracle.weight_scale(W)
            codes = oracle.ternary_codes(W, g)
            products.append(TernaryWeight(torch.from_numpy(oracle.pack(codes)),
                                          torch.tensor([g]), N, K))
            codes_all.append(codes)
            gammas.append(g)
        cpd = ColumnParallelDecode(products, M=M, device="cpu")
        # this rank's part, computed by the oracle from the shard's own bytes
        for (p, sh, sw), loc, g in zip(cpd.shards, cpd.local, gammas):
            if sw is None:
                continue
            shard_codes = oracle.unpack(sw.packed.numpy(), sw.N, K)
            bits = _oracle_y_bits(shard_codes, g, x)
            loc[:, :sh.rows] = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
        cpd.gather()
        outs = cpd.outputs()
        ok = []
        for o, codes, g in zip(outs, codes_all, gammas):
            want = _oracle_y_bits(codes, g, x)
            got = o.contiguous().view(torch.int16).numpy().view(np.uint16)
            ok.append(bool(np.array_equal(got, want)))
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(",".join(str(int(v)) for v in ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,M", [(2, 1), (3, 1), (2, 3)])
def test_gloo_ranks_gather_the_unsplit_output(tmp_path, world, M):
    # q, k, v of a 2.4B layer (scaled down in N so the oracle is quick), plus
    # a row count that leaves the last rank short
    shapes = [(256, 640), (256, 160), (256, 1001)]
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), shapes, M),
                       nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        flags = open(tmp_path / f"rank{r}.txt").read().split(",")
        assert flags == ["1"] * len(shapes), (r, flags)
