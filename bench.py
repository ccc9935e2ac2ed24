"""Benchmark of the BitNet b1.58 BitLinear decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (the decode GEMV configuration, M = 1): one decode token through the
BitLinear products of a 2.4B-parameter BitNet b1.58 model -- per layer q/o
(2560 -> 2560), k/v (2560 -> 640), gate/up (2560 -> 6912) and down
(6912 -> 2560) -- for 30 layers, every product with its own packed ternary
weight (521 MB of distinct weights per step, more than four times the 126 MB
L2, so every step streams from HBM and no flush is needed).  Each layer is
four steps of the fused GEMV (absmax int8 quantisation of x, ternary
product with int32 accumulation, rescale, bf16 out): q/k/v in one step and
gate/up in one, since each group shares its input, then o and down -- 120
steps per token.  Each step reads the output of the one before it, as in a
decoder (o reads q, gate/up read o's output, down reads gate's output, the
next layer reads down's output), so the chain is truly dependent.  Each step
is one launch with programmatic dependent launch (a launch fetches its weights
while the previous one finishes, and reads x only after it), the 120 launches
replayed from a CUDA graph captured through the public Python API.  The same
token as ONE persistent cooperative launch (DecodeChain: producer warps stream
every step's weights ahead, a software grid barrier between steps) is timed
beside it (persistent_chain, or --chain for the headline); on B200 it is the
slower of the two.  The end-to-end figure copies the token's input in and its
final output back every step.

Metric: effective weight bandwidth, packed weight bytes / device time, GB/s,
against the measured HBM copy bandwidth.  Inputs are synthetic and seeded
(weights N(0, 0.02^2) absmean-packed; x ~ N(0, 1) with 0.1% x20 outliers,
bf16).  With N GPUs every rank runs its own independent decode stream (no
collective), so the scaling is weak and the value is the sum over ranks.  With
--split the ranks share one model instead: every product is split by output
rows (whole 8-row groups of the packed weight per rank), each launch is
followed by an all-gather of its outputs, and the value is the one model's
weight bytes per step over the slowest rank's time (strong scaling).

The reference arm (--impl reference) times the CPU oracle on the host cores on
a bounded sample of the same workload.  Extra measurements (the isolated layer
shapes, the 100B-scale shapes, the binary GEMV, quantisation and the prefill
GEMM) go under "extra" in the same JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth_inputs as si  # noqa: E402

METRIC = "decode ternary GEMV effective weight GB/s (% of HBM peak); prefill int8 TOPS"
WORKLOAD = ("decode GEMV M=1, BitNet b1.58 2.4B layer shapes (q/o 2560->2560, k/v 2560->640, "
            "gate/up 2560->6912, down 6912->2560) x 30 layers, distinct packed weights per "
            "layer, fused int8 absmax quantisation, bf16 in/out; per layer 4 dependent steps "
            "(qkv, o, gate+up, down; products sharing x fused), one launch each with "
            "programmatic dependent launch")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]),
                float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured")
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def kernel_source_sha(csrc, names):
    """sha256 of the kernel's source files, concatenated in the given order."""
    import hashlib
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(chain: bool = True):
    """DRAM bytes per launch of the timed kernel from the committed ncu
    summary, or None when the kernel source has changed since those counters
    were taken."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "bit_ternary_weight_b200", "csrc")
    if chain:
        prof = os.path.join(ROOT, "profiles", "decode_chain_2b_launches.md")
        srcs = ["gemv_chain.cu", "gemv_stream_common.cuh"]
    else:
        prof = os.path.join(ROOT, "profiles", "decode_stream_2b_gemv_launches.md")
        srcs = ["gemv_stream.cu", "gemv_stream_common.cuh"]
    try:
        text = open(prof).read()
        sha = kernel_source_sha(csrc, srcs)
        m = re.search(r"sha256 prefix `([0-9a-f]+)`", text)
        t = re.search(r"traffic_per_launch_bytes: (\d+)", text)
        if m and t and sha.startswith(m.group(1)):
            return int(t.group(1))
    except OSError:
        pass
    return None


# ---------------------------------------------------------------- distributed

def dist_init(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The largest of the ranks' values (device times are reported as the max)."""
    if world == 1:
        return v
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_step_per_rank: float, steps: int, world: int, t_max: float) -> float:
    """Whole-job GB/s: every rank streams its own weights (weak scaling); the
    job takes as long as its slowest rank."""
    return bytes_per_step_per_rank * steps * world / t_max / 1e9


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of this GPU's clocks during the timed region."""

    PERIOD_MS = 100
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        self.cmd = ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}",
                    "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.15)            # nvidia-smi's start-up
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        self.out.flush()
        self.out.seek(0)
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = max(smax, float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.out.name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- workload

# One decoder layer's BitLinear launches: products that share their input are
# fused into one launch (q/k/v; gate/up), as a decoder computes them.
LAYER_LAUNCHES_2B = [("qkv", ["q", "k", "v"]), ("o", ["o"]), ("gate_up", ["gate", "up"]),
                     ("down", ["down"])]


def build_stream(bl, layers: int, seed: int, device):
    """Pack distinct weights for every product of every layer and chain the
    launches the way a decoder layer does: q/k/v read the layer input, o reads
    q, gate/up read o's output, down reads gate's output, and the next layer
    reads down's output.  Returns the launches, the token's input x0, the last
    output, the host copy of x0 and the packed bytes per step."""
    shapes = {name: (K, N) for (name, K, N) in si.LAYER_SHAPES_2B}
    gen = torch.Generator(device=device)
    per_layer = []
    total_bytes = 0
    for layer in range(layers):
        launches = []
        for li, (lname, names) in enumerate(LAYER_LAUNCHES_2B):
            ws = []
            for j, name in enumerate(names):
                K, N = shapes[name]
                gen.manual_seed(seed * 100003 + layer * 31 + li * 7 + j)
                W = torch.randn(N, K, generator=gen, device=device, dtype=torch.float32) * 0.02
                ws.append(bl.pack(W))
                del W
                total_bytes += ws[-1].packed.numel()
            launches.append(ws)
        per_layer.append(launches)
    y_elems = sum(w.N for launches in per_layer for ws in launches for w in ws)
    ys = torch.empty(y_elems, dtype=torch.bfloat16, device=device)
    x0 = torch.empty(1, si.HIDDEN_2B, dtype=torch.bfloat16, device=device)
    chain = []
    off = 0
    h = x0
    for launches in per_layer:
        outs = []
        for ws in launches:
            o = []
            for w in ws:
                o.append(ys[off:off + w.N].view(1, w.N))
                off += w.N
            outs.append(o)
        qkv, o_proj, gate_up, down = launches
        chain.append((qkv, h, outs[0]))                 # q, k, v <- layer input
        chain.append((o_proj, outs[0][0], outs[1]))     # o <- q
        chain.append((gate_up, outs[1][0], outs[2]))    # gate, up <- o
        chain.append((down, outs[2][0], outs[3]))       # down <- gate
        h = outs[3][0]
    host_x0 = si.activations(1, si.HIDDEN_2B, seed=seed)
    x0.copy_(host_x0)
    torch.cuda.synchronize()
    return chain, x0, h, host_x0, total_bytes


def run_step(bl, launches, pdl=True):
    for (ws, x, ys) in launches:
        bl.gemv_fused_multi(ws, x, outs=ys, pdl=pdl)


def build_split_stream(bl, layers: int, seed: int, device):
    """The decode stream split by output rows over the ranks (column-parallel):
    every rank packs the same model (same seeds), keeps the shard of whole
    8-row groups it owns of every weight, runs its shards of each launch and
    all-gathers the outputs, so each launch's full output is on every rank
    before the next one reads it.  Returns the per-launch ColumnParallelDecode
    objects with their inputs, the token input, the final output, the host
    token and the packed bytes per step that this rank streams and that the
    whole job streams."""
    from bit_ternary_weight_b200.sharding import ColumnParallelDecode
    shapes = {name: (K, N) for (name, K, N) in si.LAYER_SHAPES_2B}
    gen = torch.Generator(device=device)
    x0 = torch.empty(1, si.HIDDEN_2B, dtype=torch.bfloat16, device=device)
    chain = []
    h = x0
    rank_bytes = total_bytes = 0
    for layer in range(layers):
        cpds = []
        for li, (lname, names) in enumerate(LAYER_LAUNCHES_2B):
            ws = []
            for j, name in enumerate(names):
                K, N = shapes[name]
                gen.manual_seed(seed * 100003 + layer * 31 + li * 7 + j)
                W = torch.randn(N, K, generator=gen, device=device, dtype=torch.float32) * 0.02
                ws.append(bl.pack(W))
                del W
                total_bytes += ws[-1].packed.numel()
            cpd = ColumnParallelDecode(ws, device=device)
            rank_bytes += sum(sw.packed.numel() for (_, _, sw) in cpd.shards if sw is not None)
            cpds.append(cpd)
        qkv, o_proj, gate_up, down = cpds
        chain.append((qkv, h))
        chain.append((o_proj, qkv.outputs()[0]))
        chain.append((gate_up, o_proj.outputs()[0]))
        chain.append((down, gate_up.outputs()[0]))
        h = down.outputs()[0]
    host_x0 = si.activations(1, si.HIDDEN_2B, seed=seed)
    x0.copy_(host_x0)
    torch.cuda.synchronize()
    return chain, x0, h, host_x0, rank_bytes, total_bytes


def run_split_step(chain, pdl=True):
    for cpd, x in chain:
        cpd(x, pdl=pdl)


def load_replays(graph, n: int):
    """n untimed replays of the step's graph, then a synchronize: the same load
    as the timed steps, for the clock samples around them."""
    for _ in range(n):
        graph.replay()
    torch.cuda.synchronize()


def time_graph(graph, steps, world):
    barrier(world)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        graph.replay()
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end) / 1000.0


def isolated_gemv(bl, K, N, M=1, iters=200, copies=None, device="cuda", pdl=False,
                  force_fused=None, small_batch="auto", ws=None):
    """Per-launch time of one shape, rotating distinct weight copies (>= 4x L2).

    pdl: consecutive launches (M = 1) overlap through programmatic dependent
    launch, as consecutive GEMVs of a decode step do; each still reads x only
    after the previous launch has finished.  small_batch: for 2 .. 16 tokens,
    "auto", "tensor" or "dp4a" (the kernel the fused call runs).  ws: the
    rotated weight copies, built here when not given."""
    nbytes = bl.packed_bytes(N, K)
    if ws is None:
        if copies is None:
            copies = max(2, int((4 * 126e6) // nbytes) + 1)
        ws = _weight_copies(bl, K, N, nbytes, 7, device, limit=min(copies, 400))
    copies = len(ws)
    x = si.activations(M, K, seed=5).to(device)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
    # the path bl.linear takes: a fused GEMV for few tokens, else quantise +
    # tensor-core GEMM (both launches timed)
    fused = bl.fused_gemv_preferred(M, N, K) if force_fused is None else force_fused
    if fused:
        call = lambda wt: bl.gemv_fused_multi([wt], x, outs=[y], pdl=pdl, small_batch=small_batch)  # noqa: E731
    else:
        q = torch.empty(M, K, dtype=torch.int8, device=device)
        d = torch.empty(M, dtype=torch.float32, device=device)
        r = torch.empty(M, dtype=torch.int32, device=device)
        # split-K workspace: zero once, left zero by every call
        gws = torch.zeros(max(bl.gemm_workspace_bytes(M, N, K), 16), dtype=torch.uint8, device=device)

        def call(wt):
            bl.quantize_act(x, out=(q, d, r))
            bl.gemm(wt, q, d, r, out=y, workspace=gws)
    for i in range(min(copies, 8)):
        call(ws[i])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(iters):
            call(ws[i % copies])
    g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    g.replay()
    e.record()
    torch.cuda.synchronize()
    t = s.elapsed_time(e) / 1000.0 / iters
    del g
    return {"K": K, "N": N, "M": M, "us": t * 1e6, "GBps": nbytes / t / 1e9,
            "weight_copies": copies, "pdl": pdl,
            "path": gemv_path(bl, K, N, M, fused, small_batch)}


def gemv_path(bl, K, N, M, fused, small_batch="auto"):
    """Which kernel the library runs for this shape (the library's own plan)."""
    if not fused:
        return "quantise + tcgen05 GEMM"
    kern, cluster = bl.gemv_plan([N], K, M, small_batch=small_batch)
    return {"stream": "fused streaming GEMV (producer warp, bulk copies, mbarrier ring)",
            "tensor": f"tensor-core small-batch GEMV (clusters of {cluster} CTAs per 128-row block)",
            "stream_mt": "fused multi-token streaming GEMV (dp4a, one weight pass for all tokens)",
            "dp4a": "fused dp4a GEMV (per-warp cp.async ring)"}[kern]


def small_batch_sweep(bl, device="cuda"):
    """Config 3's timing: M in {1, 2, 4, 8, 16} on the four 2.4B shapes.
    `us` / `GBps` / `path` are what linear() runs (the library's routing); from
    2 tokens the two small-batch kernels are timed side by side (`tensor_us`,
    `dp4a_us`) and from 8 tokens also quantise + GEMM (`gemm_us`); `pdl_us` is
    what linear() runs with consecutive launches overlapping through
    programmatic dependent launch, as consecutive layers of a decode step do."""
    out = []
    for (K, N) in si.DECODE_SHAPES_2B:
        nbytes = bl.packed_bytes(N, K)
        ws = _weight_copies(bl, K, N, nbytes, 7, device)
        for m in si.SMALL_BATCH_M:
            r = dict(isolated_gemv(bl, K, N, M=m, iters=100, device=device, ws=ws))
            if m >= 2:
                r["tensor_us"] = isolated_gemv(bl, K, N, M=m, iters=100, device=device, force_fused=True,
                                               small_batch="tensor", ws=ws)["us"]
                r["dp4a_us"] = isolated_gemv(bl, K, N, M=m, iters=100, device=device, force_fused=True,
                                             small_batch="dp4a", ws=ws)["us"]
                r["pdl_us"] = isolated_gemv(bl, K, N, M=m, iters=100, device=device, pdl=True,
                                            ws=ws)["us"]
            if m >= 8:
                r["gemm_us"] = isolated_gemv(bl, K, N, M=m, iters=100, device=device, force_fused=False,
                                             ws=ws)["us"]
            out.append(r)
        del ws
    return out


def isolated_binary(bl, K, N, iters=100, device="cuda"):
    nbytes = N * K // 8
    copies = max(2, int((4 * 126e6) // nbytes) + 1)
    gen = torch.Generator(device=device)
    ws = []
    for c in range(copies):
        gen.manual_seed(11 + c)
        W = torch.randn(N, K, generator=gen, device=device) * 0.02
        ws.append(bl.binary_pack(W))
        del W
    x = si.activations(1, K, seed=5).to(device)
    y = torch.empty(N, dtype=torch.bfloat16, device=device)
    bl.binary_gemv(ws[0], x, out=y)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(iters):
            bl.binary_gemv(ws[i % copies], x, out=y)
    g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    g.replay()
    e.record()
    torch.cuda.synchronize()
    t = s.elapsed_time(e) / 1000.0 / iters
    del g, ws
    return {"K": K, "N": N, "us": t * 1e6, "GBps": nbytes / t / 1e9, "weight_copies": copies}


def _graph_time(calls, iters):
    """Per-call device time of `calls` (a list of thunks, cycled) replayed
    from one CUDA graph of `iters` launches."""
    for c in calls[:min(len(calls), 4)]:
        c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(iters):
            calls[i % len(calls)]()
    g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    g.replay()
    e.record()
    torch.cuda.synchronize()
    del g
    return s.elapsed_time(e) / 1000.0 / iters


def _weight_copies(bl, K, N, nbytes, seed0, device, limit=400):
    copies = min(limit, max(2, int((4 * 126e6) // nbytes) + 1))
    gen = torch.Generator(device=device)
    ws = []
    for c in range(copies):
        gen.manual_seed(seed0 + c)
        W = torch.randn(N, K, generator=gen, device=device) * 0.02
        ws.append(bl.pack(W))
        del W
    return ws


def isolated_bitplane(bl, K, N, iters=100, device="cuda"):
    """Ternary x 1-bit bit-plane GEMV (N*K/4 bytes of planes), weights
    rotated beyond L2."""
    nbytes = N * K // 4
    ws = [bl.bitplane_pack(w) for w in _weight_copies(bl, K, N, nbytes, 13, device)]
    x = si.activations(1, K, seed=5).to(device)
    y = torch.empty(N, dtype=torch.bfloat16, device=device)
    t = _graph_time([lambda w=w: bl.bitplane_gemv(w, x, out=y) for w in ws], iters)
    return {"K": K, "N": N, "us": t * 1e6, "GBps": nbytes / t / 1e9, "weight_copies": len(ws)}


def lut_vs_dp4a(bl, K, N, iters=100, device="cuda"):
    """Table-lookup GEMV against the dp4a GEMV on the same pre-quantised token
    and the same rotated weights."""
    nbytes = bl.packed_bytes(N, K)
    ws = _weight_copies(bl, K, N, nbytes, 17, device)
    x = si.activations(1, K, seed=5).to(device)
    q, d, r = bl.quantize_act(x)
    y = torch.empty(1, N, dtype=torch.bfloat16, device=device)
    t_lut = _graph_time([lambda w=w: bl.lut_gemv(w, q, d, out=y) for w in ws], iters)
    t_dp4a = _graph_time([lambda w=w: bl.gemv(w, q, d, r, out=y) for w in ws], iters)
    return {"K": K, "N": N, "lut_us": t_lut * 1e6, "lut_GBps": nbytes / t_lut / 1e9,
            "dp4a_us": t_dp4a * 1e6, "dp4a_GBps": nbytes / t_dp4a / 1e9,
            "weight_copies": len(ws)}


def rmsnorm_gemv_cost(bl, K, Ns, iters=200, device="cuda"):
    """RMSNorm + quantise + products sharing the token in one launch, against
    the same launch without RMSNorm (same rotated weights)."""
    per = sum(bl.packed_bytes(N, K) for N in Ns)
    sets = []
    for c in range(min(400, max(2, int((4 * 126e6) // per) + 1))):
        gen = torch.Generator(device=device)
        gen.manual_seed(23 + c)
        sets.append([bl.pack(torch.randn(N, K, generator=gen, device=device) * 0.02) for N in Ns])
    x = si.activations(1, K, seed=5).to(device)
    gain = (1.0 + 0.1 * torch.randn(K, device=device)).to(torch.bfloat16)
    outs = [torch.empty(1, N, dtype=torch.bfloat16, device=device) for N in Ns]
    t_norm = _graph_time([lambda ws=ws: bl.rmsnorm_gemv_fused_multi(ws, x, gain, outs=outs)
                          for ws in sets], iters)
    t_plain = _graph_time([lambda ws=ws: bl.gemv_fused_multi(ws, x, outs=outs) for ws in sets], iters)
    return {"K": K, "N": Ns, "rmsnorm_us": t_norm * 1e6, "plain_us": t_plain * 1e6,
            "rmsnorm_GBps": per / t_norm / 1e9, "plain_GBps": per / t_plain / 1e9}


def decoder_tokens(bl, contexts=(512, 2048), tokens=64, device="cuda"):
    """The synthetic 2.4B decoder stack (30 layers: RMSNorm, q/k/v, RoPE +
    attention over a bf16 KV cache, o + residual, RMSNorm, gate/up, squared
    ReLU gate, down + residual; 151 launches per token with PDL) replayed
    from a CUDA graph, one token per replay, at a given number of cached
    positions."""
    from bit_ternary_weight_b200.decoder import Decoder, DecoderConfig
    cfg = DecoderConfig(max_seq=max(contexts) + tokens + 8)
    dec = Decoder.random(cfg, seed=1, device=device)
    dec.h.copy_(si.activations(1, cfg.hidden, seed=5)[0])
    out = []
    dec.set_position(0)
    dec.step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dec.step()
    for ctx in contexts:
        dec.set_position(ctx)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(tokens):
            g.replay()
        e.record()
        torch.cuda.synchronize()
        t = s.elapsed_time(e) / 1000.0 / tokens
        out.append({"context": ctx, "tokens": tokens, "us_per_token": t * 1e6,
                    "tokens_per_s": 1.0 / t, "weight_GBps": dec.weight_bytes() / t / 1e9,
                    "launches_per_token": 5 * cfg.layers + 1})
    assert bl.last_device_status() == 0
    del g, dec
    return out


def prefill_gemm(bl, K, N, M, iters=20, device="cuda"):
    gen = torch.Generator(device=device)
    gen.manual_seed(3)
    W = torch.randn(N, K, generator=gen, device=device) * 0.02
    w = bl.pack(W)
    del W
    x = (torch.randn(M, K, generator=gen, device=device)).to(torch.bfloat16)
    q, d, r = bl.quantize_act(x)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
    ws = torch.empty(max(bl.gemm_workspace_bytes(M, N, K), 16), dtype=torch.uint8, device=device)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    bl.gemm(w, q, d, r, out=y, workspace=ws)
    torch.cuda.synchronize()
    gain = (1.0 + 0.1 * torch.randn(K, generator=gen, device=device)).to(torch.bfloat16)
    times, qtimes, ntimes = [], [], []
    for _ in range(iters):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        bl.gemm(w, q, d, r, out=y, workspace=ws)
        e.record()
        flush.zero_()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record()
        bl.quantize_act(x, out=(q, d, r))
        e2.record()
        flush.zero_()
        s3, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s3.record()
        bl.rmsnorm_quantize_act(x, gain, out=(q, d, r))
        e3.record()
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e) / 1000.0)
        qtimes.append(s2.elapsed_time(e2) / 1000.0)
        ntimes.append(s3.elapsed_time(e3) / 1000.0)
    t = statistics.median(times)
    tq = statistics.median(qtimes)
    tn = statistics.median(ntimes)
    ops = 2.0 * M * N * K
    return {"M": M, "K": K, "N": N, "gemm_us": t * 1e6, "TOPS": ops / t / 1e12,
            "quant_us": tq * 1e6, "quant_GBps": M * K * 3 / tq / 1e9,
            "rmsnorm_quant_us": tn * 1e6, "rmsnorm_quant_GBps": M * K * 3 / tn / 1e9,
            "TOPS_incl_quant": ops / (t + tq) / 1e12}


# ---------------------------------------------------------------- CPU oracle leg

def oracle_sample(seconds_target: float, seed: int = 0):
    """Time the oracle on layers of the same workload; returns GB/s and details."""
    import numpy as np
    import oracle
    layer = []
    for j, (name, K, N) in enumerate(si.LAYER_SHAPES_2B):
        W = si.weight(N, K, seed=seed * 100 + j).numpy()
        g = oracle.weight_scale(W)
        codes = oracle.ternary_codes(W, g)
        x = si.activations(1, K, seed=seed + j).float().numpy()
        layer.append((K, N, g, codes, x))
    per_layer_bytes = sum(oracle.packed_bytes(N, K) for (K, N, _, _, _) in layer)
    done = 0
    t0 = time.perf_counter()
    while True:
        for (K, N, g, codes, x) in layer:
            q, d, r = oracle.quantize_act(x)
            acc = oracle.ternary_acc(codes, q)
            y = oracle.rescale(acc, d, g)
            oracle.to_bf16_bits(y)
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds_target:
            break
    _ = np  # numpy imported for the oracle's arrays
    return {"value": per_layer_bytes * done / el / 1e9, "unit": "GB/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{done} passes over one layer's 7 BitLinear products "
                      f"({per_layer_bytes / 1e6:.1f} MB of packed weights each), "
                      f"{el:.1f} s of CPU work",
            "seconds": el, "layers": done}


def oracle_prefill_sample(M: int = 64, K: int = 2560, N: int = 6912, runs: int = 3, seed: int = 0):
    """Time the oracle's prefill product (quantise, accumulate, rescale) on M tokens; best of runs."""
    import oracle
    W = si.weight(N, K, seed=seed).numpy()
    g = oracle.weight_scale(W)
    codes = oracle.ternary_codes(W, g)
    x = si.activations(M, K, seed=seed + 1).float().numpy()
    best = None
    for _ in range(runs):
        t0 = time.perf_counter()
        q, d, r = oracle.quantize_act(x)
        acc = oracle.ternary_acc(codes, q)
        y = oracle.rescale(acc, d, g)
        oracle.to_bf16_bits(y)
        el = time.perf_counter() - t0
        best = el if best is None else min(best, el)
    return {"TOPS": 2.0 * M * N * K / best / 1e12, "M": M, "K": K, "N": N,
            "seconds_best": best, "runs": runs, "cores": oracle.num_threads()}


def cpu_baseline(seconds: float):
    """The oracle on the host cores: best of 3 samples on all cores, one on one core, prefill."""
    import oracle
    all_cores = oracle.num_threads()
    part = seconds / 5.0
    runs = [oracle_sample(part, seed=0) for _ in range(3)]
    best = max(runs, key=lambda r: r["value"])
    oracle.set_num_threads(1)
    try:
        one = oracle_sample(part, seed=0)
    finally:
        oracle.set_num_threads(all_cores)
    prefill = oracle_prefill_sample()
    return {"value": best["value"], "unit": "GB/s", "cores": best["cores"], "kind": "oracle",
            "sample": best["sample"] + "; best of 3 such samples",
            "runs_GBps": [r["value"] for r in runs],
            "one_core": {"value": one["value"], "unit": "GB/s", "cores": one["cores"],
                         "sample": one["sample"]},
            "prefill": prefill, "cpu": cpu_model()}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


# ---------------------------------------------------------------- arms

def run_reference(args, world, rank):
    if rank != 0:
        return
    res = None
    for _ in range(args.warmup):
        oracle_sample(0.0, seed=1)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        res = oracle_sample(args.ref_seconds, seed=0)
        vals.append(res["value"])
    el = time.perf_counter() - t0
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / max(1, args.steps) * 1000, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": "CPU oracle, bounded sample per step"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": res["cores"],
                         "kind": "oracle", "sample": res["sample"], "cpu": cpu_model()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    import bit_ternary_weight_b200 as bl
    device = torch.device("cuda", torch.cuda.current_device())
    hbm, bf16, bf16_sus, peak_kind = peaks()

    if args.split:
        # one model split over the ranks: every rank builds it from the same seed
        launches, xs, ys, host_x, rank_bytes, step_bytes = build_split_stream(
            bl, args.layers, seed=0, device=device)
        step = lambda: run_split_step(launches)  # noqa: E731
    else:
        launches, xs, ys, host_x, step_bytes = build_stream(bl, args.layers, seed=rank, device=device)
        rank_bytes = step_bytes
        if args.chain:
            # the token's whole chain in one persistent launch
            chain = bl.DecodeChain([bl.ChainStep(ws, x, outs) for (ws, x, outs) in launches])
            step = chain.run
        else:
            step = lambda: run_step(bl, launches)  # noqa: E731
    # xs: the token's input (copied in every e2e step); ys: its final output
    products_per_step = len(launches)
    kernel_launches_per_step = 1 if (args.chain and not args.split) else products_per_step
    # eager warm-up through the public API, then capture the step
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    # the timed steps last milliseconds, far less than nvidia-smi's sampling
    # period, so the same replays run for ~0.5 s on either side of them (each
    # side ended by a synchronize; the timed steps keep their own barrier and
    # synchronize on both sides) and the samples see the clocks under this
    # load.  The replay count is agreed over the ranks: a split step's graph
    # holds collectives, so every rank must replay it equally often.
    t_est = max_over_ranks(time_graph(graph, args.warmup, world) / args.warmup, world)
    n_load = max(1, min(100000, int(0.5 / max(t_est, 1e-6))))
    with ClockSampler(local) as clk:
        load_replays(graph, n_load)
        t = time_graph(graph, args.steps, world)
        load_replays(graph, n_load)
    clocks = clk.summary()
    clocks["how"] = (f"nvidia-smi every {ClockSampler.PERIOD_MS} ms while the step's graph "
                     f"replays {n_load} times (~0.5 s) on each side of the timed steps")
    t = max_over_ranks(t, world)
    # replicas: every rank streams a whole model per step (weak scaling);
    # split: the ranks stream one model between them (strong scaling)
    job_ranks = 1 if args.split else world
    value = job_throughput(step_bytes, args.steps, job_ranks, t)
    ms_per_step = t / args.steps * 1000

    # e2e: host activations in, host outputs back, every step, through the same
    # public-API launches (replayed from the graph captured above)
    pin_x = host_x.pin_memory()
    pin_y = torch.empty(ys.shape, dtype=ys.dtype).pin_memory()
    for _ in range(3):
        xs.copy_(pin_x, non_blocking=True)
        graph.replay()
        pin_y.copy_(ys, non_blocking=True)
    barrier(world)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.steps):
        xs.copy_(pin_x, non_blocking=True)
        graph.replay()
        pin_y.copy_(ys, non_blocking=True)
    e.record()
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(s.elapsed_time(e) / 1000.0, world)
    e2e_value = job_throughput(step_bytes, args.steps, job_ranks, t_e2e)

    # eager (no graph) public-API loop, for context
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    eager_steps = max(1, min(args.steps, 20))
    s.record()
    for _ in range(eager_steps):
        xs.copy_(pin_x, non_blocking=True)
        step()
        pin_y.copy_(ys, non_blocking=True)
    e.record()
    torch.cuda.synchronize()
    t_eager = s.elapsed_time(e) / 1000.0
    del graph

    # the same token as ONE persistent launch (DecodeChain), for comparison
    other = None
    if not args.split and not args.chain:
        chain = bl.DecodeChain([bl.ChainStep(ws, x, outs) for (ws, x, outs) in launches])
        chain.run()
        torch.cuda.synchronize()
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            chain.run()
        for _ in range(args.warmup):
            g2.replay()
        t_ch = max_over_ranks(time_graph(g2, args.steps, world), world)
        other = {"GBps": job_throughput(step_bytes, args.steps, world, t_ch),
                 "ms_per_step": t_ch / args.steps * 1000, "launches_per_step": 1,
                 "how": "DecodeChain: the token's 120 steps in one persistent cooperative "
                        "launch (software grid barrier per step), CUDA graph"}
        del g2

    extra = {}
    if rank == 0 and not args.no_extra and not args.split:
        def measure(key, fn):
            try:
                extra[key] = fn()
            except Exception as ex:  # reported in the line, never hidden
                extra[key] = {"error": str(ex)[:300]}
        measure("isolated_2b", lambda: [isolated_gemv(bl, K, N, device=device)
                                        for (K, N) in si.DECODE_SHAPES_2B])
        measure("isolated_100b", lambda: [isolated_gemv(bl, K, N, iters=200, device=device)
                                          for (K, N) in si.DECODE_SHAPES_100B])
        measure("chained_100b_pdl", lambda: [isolated_gemv(bl, K, N, iters=200, device=device, pdl=True)
                                             for (K, N) in si.DECODE_SHAPES_100B])
        measure("small_batch", lambda: small_batch_sweep(bl, device=device))
        measure("binary_100b", lambda: isolated_binary(bl, 8192, 28672, device=device))
        measure("bitplane_100b", lambda: [isolated_bitplane(bl, K, N, device=device)
                                          for (K, N) in si.DECODE_SHAPES_100B])
        measure("lut_vs_dp4a", lambda: [lut_vs_dp4a(bl, K, N, device=device)
                                        for (K, N) in si.DECODE_SHAPES_2B + [(8192, 28672)]])
        measure("decoder_2b", lambda: decoder_tokens(bl, device=device))
        measure("rmsnorm_gemv", lambda: [rmsnorm_gemv_cost(bl, 2560, [6912, 6912], device=device),
                                         rmsnorm_gemv_cost(bl, 2560, [2560, 640, 640], device=device),
                                         rmsnorm_gemv_cost(bl, 8192, [28672], device=device)])
        measure("mma_peak", lambda: bl.probe_mma_i8(device=device))
        measure("prefill", lambda: [prefill_gemm(bl, K, N, M, device=device)
                                    for (K, N) in si.PREFILL_SHAPES for M in si.PREFILL_TOKENS])
        probe = extra.get("mma_peak", {}).get("tops")
        for r in extra.get("prefill", []) if isinstance(extra.get("prefill"), list) else []:
            r["roofline"] = {"bound": "tensor", "achieved": r["TOPS"], "unit": "TOPS",
                             "peak_2x_bf16": 2 * bf16, "frac_2x_bf16": r["TOPS"] / (2 * bf16),
                             "peak_probe": probe,
                             "frac_probe": r["TOPS"] / probe if probe else None,
                             "peak_kind": f"2 x {peak_kind} bf16 cuBLAS burst (nominal int8/bf16 "
                                          "ratio); probe: back-to-back tcgen05.mma.kind::i8 of "
                                          "the GEMM's form (bitlinear_probe_mma_i8)"}

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_seconds)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "strong" if args.split else "weak",
        "vs_baseline": None,
        "dtype": "int8", "data": "synthetic (seeded N(0,0.02) weights, N(0,1) bf16 x with 0.1% x20 outliers)",
        "config": {"workload": WORKLOAD, "layers": args.layers,
                   "products_per_step": products_per_step,
                   "launches_per_step": kernel_launches_per_step,
                   "weight_bytes_per_step": step_bytes,
                   "weight_bytes_per_step_per_rank": rank_bytes,
                   "l2": "inputs larger than L2: 521 MB of distinct packed weights per step",
                   "parallelism": (f"N-split over {world} ranks (each launch's output rows "
                                   "split in whole 8-row groups, all-gather of y after every "
                                   "launch)") if args.split else
                                  f"{world} independent replicas (weak scaling)"},
        "roofline": {"bound": "hbm", "achieved": rank_bytes * args.steps / t / 1e9, "peak": hbm,
                     "unit": "GB/s", "frac": rank_bytes * args.steps / t / 1e9 / hbm,
                     "traffic": profiled_traffic(chain=kernel_launches_per_step == 1),
                     "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "kernel": ("gemv_chain_kernel (one persistent launch per token)"
                                if kernel_launches_per_step == 1 else
                                "gemv_stream_kernel<KC=10, bf16 fused> (4 launches per layer)"),
                     "note": "algorithmic bytes = packed weight bytes per launch; duration = "
                             "step time / launches per step (CUDA events over the timed "
                             "region, on the launching stream)"},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "GB/s",
                "h2d_bytes_per_step": xs.numel() * xs.element_size(),
                "d2h_bytes_per_step": ys.numel() * ys.element_size(),
                "how": "pinned host token input -> device, graph of the public-API "
                       "gemv_fused_multi chain, final output -> pinned host, CUDA events"},
        "e2e_eager_GBps": step_bytes * eager_steps / t_eager / 1e9,
        "persistent_chain": other,
        "gpu_launches": kernel_launches_per_step * args.steps,
        "clocks": clocks,
        "extra": extra,
    }
    print(json.dumps(line), flush=True)


def run_case(args):
    """One kernel on one shape, --iters times (for profiling); prints a JSON line."""
    import bit_ternary_weight_b200 as bl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(17)
    K, N, M = args.K, args.N, args.M
    W = torch.randn(N, K, generator=gen, device=dev) * 0.02
    x = si.activations(M, K, seed=9).to(dev)
    if args.case == "binary":
        w = bl.binary_pack(W)
        fn = lambda: bl.binary_gemv(w, x[0])  # noqa: E731
        nbytes, ops = N * K // 8, 2 * N * K
    elif args.case == "bitplane":
        w = bl.bitplane_pack(bl.pack(W))
        fn = lambda: bl.bitplane_gemv(w, x[0])  # noqa: E731
        nbytes, ops = N * K // 4, 2 * N * K
    elif args.case == "lut":
        w = bl.pack(W)
        q, d, _ = bl.quantize_act(x[:1])
        fn = lambda: bl.lut_gemv(w, q, d)  # noqa: E731
        nbytes, ops = bl.packed_bytes(N, K), 2 * N * K
    else:
        w = bl.pack(W)
        if args.case == "gemv":
            y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            fn = lambda: bl.gemv_fused_multi([w], x, outs=[y], small_batch=args.small_batch)  # noqa: E731
        else:
            q, d, r = bl.quantize_act(x)
            ws = torch.zeros(max(bl.gemm_workspace_bytes(M, N, K), 16), dtype=torch.uint8, device=dev)
            fn = lambda: bl.gemm(w, q, d, r, workspace=ws)  # noqa: E731
        nbytes, ops = bl.packed_bytes(N, K), 2 * M * N * K
    del W
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.iters):
        fn()
    e.record()
    torch.cuda.synchronize()
    t = s.elapsed_time(e) / 1000.0 / args.iters
    line = {"case": args.case, "K": K, "N": N, "M": M, "iters": args.iters,
            "us": t * 1e6, "weight_GBps": nbytes / t / 1e9, "TOPS": ops / t / 1e12,
            "note": "same weights every launch (L2-warm unless profiled)"}
    if args.case == "gemv":
        line["kernel"] = list(bl.gemv_plan([N], K, M, small_batch=args.small_batch))
    print(json.dumps(line), flush=True)


def run_decoder_case(args):
    """The synthetic decoder stack, eager (no graph), `--iters` tokens from
    `--ctx` cached positions with `--layers` layers: for launch lists and
    per-launch profiles of one token's kernels; prints one JSON line."""
    import bit_ternary_weight_b200 as bl  # noqa: F401  (loads the library)
    from bit_ternary_weight_b200.decoder import Decoder, DecoderConfig
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = DecoderConfig(layers=args.layers, max_seq=args.ctx + args.iters + 8)
    dec = Decoder.random(cfg, seed=1, device=dev)
    dec.h.copy_(si.activations(1, cfg.hidden, seed=5)[0])
    dec.set_position(args.ctx)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.iters):
        dec.step()
    e.record()
    torch.cuda.synchronize()
    print(json.dumps({"case": "decoder", "layers": args.layers, "context": args.ctx, "tokens": args.iters,
                      "us_per_token_eager": s.elapsed_time(e) * 1000.0 / args.iters,
                      "launches_per_token": 5 * args.layers + 1}), flush=True)


def run_mma_peak(args):
    """The int8 tensor-core rate of the prefill GEMM's MMA form, with the SM
    clocks sampled while it runs; prints one JSON line."""
    import bit_ternary_weight_b200 as bl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    bl.probe_mma_i8(reps=1000, device=dev)                 # warm-up
    with ClockSampler(0) as clk:
        runs = [bl.probe_mma_i8(reps=100000, device=dev) for _ in range(max(3, args.iters))]
        # narrow MMAs (the small-batch GEMV's 128 x 32 x 32) from 1, 2 and 4 issuing warps
        issue = [min((bl.probe_mma_i8(reps=50000, device=dev, n=32, issuers=w) for _ in range(3)),
                     key=lambda r: r["cycles_per_mma_per_sm"]) for w in (1, 2, 4)]
    best = max(runs, key=lambda r: r["tops"])
    print(json.dumps({"case": "mma_peak", "mac_per_clk_per_sm": best["mac_per_clk_per_sm"],
                      "tops": best["tops"], "ctas": best["ctas"], "runs": len(runs),
                      "cycles_per_mma_per_sm": best["cycles_per_mma_per_sm"],
                      "narrow_mma_issue": [{"n": r["n"], "issuers": r["issuers"],
                                            "cycles_per_mma_per_sm": r["cycles_per_mma_per_sm"],
                                            "mac_per_clk_per_sm": r["mac_per_clk_per_sm"]} for r in issue],
                      "clocks": clk.summary(),
                      "note": "back-to-back tcgen05.mma.kind::i8 128x128x32 (A in TMEM, B in "
                              "swizzled smem), no operand traffic, one CTA per SM; narrow_mma_issue: "
                              "128x32x32 from 1, 2, 4 warps at once, each its own accumulator"}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=["stream", "gemv", "gemm", "binary", "bitplane", "lut", "mma_peak",
                                       "decoder"],
                    default="stream",
                    help="stream: the benchmark; others: one kernel on one shape (profiling)")
    ap.add_argument("--K", type=int, default=8192)
    ap.add_argument("--N", type=int, default=28672)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--iters", type=int, default=5)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=si.LAYERS_2B)
    ap.add_argument("--ctx", type=int, default=512, help="--case decoder: cached positions")
    ap.add_argument("--small-batch", choices=["auto", "tensor", "dp4a"], default="auto",
                    help="--case gemv with 2..16 tokens: the small-batch kernel to run")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=2.0)
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--chain", action="store_true",
                    help="time the step as one persistent launch (DecodeChain) instead of "
                         "one launch per product with programmatic dependent launch")
    ap.add_argument("--split", action="store_true",
                    help="split one model's products by output rows over the ranks "
                         "(column-parallel, all-gather of y per launch) instead of "
                         "running independent replicas")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.case == "mma_peak":
        run_mma_peak(args)
        return
    if args.case == "decoder":
        run_decoder_case(args)
        return
    if args.case != "stream":
        run_case(args)
        return
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_init(args.gpus)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
