"""Host-side checks of the C ABI that need no GPU.

The library must load and export every function that include/*.h declares;
argument errors (null pointers, element types, shapes, alignment) must be
reported with the documented status before any CUDA call, so they are
testable on a machine without a device.
"""
import ctypes
import glob
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(bitlinear_\w+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def bl():
    import bit_ternary_weight_b200 as b
    return b


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("bitlinear_pack", "bitlinear_quantize_act", "bitlinear_gemv",
                     "bitlinear_gemm", "bitlinear_binary_gemv"):
        assert required in names


def test_every_declared_symbol_is_exported(bl):
    raw = ctypes.CDLL(bl.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(raw, n)]
    assert not missing, missing


def test_status_strings(bl):
    for s in range(10):
        assert bl.lib.bitlinear_status_string(s).startswith(b"BL_")
    assert bl.lib.bitlinear_status_string(99) == b"unknown status"


@pytest.mark.parametrize("N,K", [(1, 64), (8, 128), (13, 256), (640, 2560), (28672, 8192),
                                 (8192, 28672)])
def test_packed_sizes_match_layout(bl, N, K):
    assert bl.packed_bytes(N, K) == oracle.packed_bytes(N, K)
    assert bl.lib.bitlinear_binary_packed_bytes(N, K) == N * (K // 64) * 8
    assert bl.lib.bitlinear_pack_workspace_bytes(N, K) == 8 * N


@pytest.mark.parametrize("N,K", [(0, 64), (8, 0), (8, 100), (8, 32), (-1, 64)])
def test_invalid_shapes_have_no_size(bl, N, K):
    assert bl.packed_bytes(N, K) == 0
    assert bl.lib.bitlinear_binary_packed_bytes(N, K) == 0


# Fake device addresses: the argument checks must reject these calls before any
# CUDA call, so the pointers are never dereferenced.
A = 0x7f0000000000          # 16-byte aligned
MIS = A + 4                 # misaligned for 16-byte vectors


def _gemv(bl, packed=A, scale=A, N=256, K=256, q=A, d=A, r=A, M=1, y=A, yt=1, ldy=256,
          acc=None):
    return bl.lib.bitlinear_gemv(packed, scale, N, K, q, d, r, M, y, yt, ldy, acc, None)


def test_gemv_argument_errors(bl):
    assert _gemv(bl, packed=None) == bl.BL_ERR_NULL
    assert _gemv(bl, q=None) == bl.BL_ERR_NULL
    assert _gemv(bl, y=None) == bl.BL_ERR_NULL
    assert _gemv(bl, yt=7) == bl.BL_ERR_DTYPE
    assert _gemv(bl, K=100) == bl.BL_ERR_SHAPE
    assert _gemv(bl, M=0) == bl.BL_ERR_SHAPE
    assert _gemv(bl, M=17) == bl.BL_ERR_SHAPE
    assert _gemv(bl, ldy=10) == bl.BL_ERR_SHAPE
    assert _gemv(bl, M=16, K=16384) == bl.BL_ERR_SHAPE  # activations exceed on-chip staging
    assert _gemv(bl, packed=MIS) == bl.BL_ERR_ALIGN
    assert _gemv(bl, q=MIS) == bl.BL_ERR_ALIGN


def test_fused_and_quant_argument_errors(bl):
    L = bl.lib
    assert L.bitlinear_gemv_fused(A, A, 256, 256, None, 1, 256, 1, A, 1, 256, None, None) == bl.BL_ERR_NULL
    assert L.bitlinear_gemv_fused(A, A, 256, 256, A, 5, 256, 1, A, 1, 256, None, None) == bl.BL_ERR_DTYPE
    assert L.bitlinear_gemv_fused(A, A, 256, 256, A, 1, 100, 1, A, 1, 256, None, None) == bl.BL_ERR_SHAPE
    # ldx of 260 bf16 elements = 520 bytes: rows not 16-byte aligned
    assert L.bitlinear_gemv_fused(A, A, 256, 256, A, 1, 260, 1, A, 1, 256, None, None) == bl.BL_ERR_ALIGN
    assert L.bitlinear_quantize_act(None, 1, 4, 256, 256, A, A, A, None) == bl.BL_ERR_NULL
    assert L.bitlinear_quantize_act(A, 3, 4, 256, 256, A, A, A, None) == bl.BL_ERR_DTYPE
    assert L.bitlinear_quantize_act(A, 1, 0, 256, 256, A, A, A, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_quantize_act(A, 1, 4, 256, 128, A, A, A, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_quantize_act(MIS, 1, 4, 256, 256, A, A, A, None) == bl.BL_ERR_ALIGN


def test_pack_and_binary_argument_errors(bl):
    L = bl.lib
    assert L.bitlinear_pack(None, 0, 8, 64, A, A, A, 64, None) == bl.BL_ERR_NULL
    assert L.bitlinear_pack(A, 2, 8, 64, A, A, A, 64, None) == bl.BL_ERR_DTYPE
    assert L.bitlinear_pack(A, 0, 8, 96, A, A, A, 64, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_pack(MIS, 0, 8, 64, A, A, A, 64, None) == bl.BL_ERR_ALIGN
    assert L.bitlinear_binary_pack(A, 0, 8, 64, None, A, None) == bl.BL_ERR_NULL
    assert L.bitlinear_binary_gemv(A, A, 8, 64, A, 9, A, 1, None, None) == bl.BL_ERR_DTYPE
    assert L.bitlinear_binary_gemv(A, A, 8, 65, A, 1, A, 1, None, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_gemm(A, A, 8, 64, None, A, A, 4, A, 1, 8, None, None, 0, None) == bl.BL_ERR_NULL
    assert L.bitlinear_gemm(A, A, 8, 64, A, A, A, 0, A, 1, 8, None, None, 0, None) == bl.BL_ERR_SHAPE


def test_valid_arguments_without_device_fail_cleanly(bl):
    """On a machine with no GPU the checks pass and the device query fails."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    st = _gemv(bl)
    assert st in (bl.BL_ERR_CUDA, bl.BL_ERR_UNSUPPORTED)


def test_rmsnorm_argument_errors_before_any_cuda_call(bl):
    A = 0x7f0000000000
    L = bl.lib
    # null, dtype, shape (negative / non-finite eps, K), alignment
    assert L.bitlinear_rmsnorm_quantize_act(None, 1, 1, 64, 64, None, 0, 1e-5, A, A, A, None) == bl.BL_ERR_NULL
    assert L.bitlinear_rmsnorm_quantize_act(A, 7, 1, 64, 64, None, 0, 1e-5, A, A, A, None) == bl.BL_ERR_DTYPE
    assert L.bitlinear_rmsnorm_quantize_act(A, 1, 1, 64, 64, A, 5, 1e-5, A, A, A, None) == bl.BL_ERR_DTYPE
    assert L.bitlinear_rmsnorm_quantize_act(A, 1, 1, 64, 64, None, 0, -1.0, A, A, A, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_rmsnorm_quantize_act(A, 1, 1, 64, 64, None, 0, float("nan"), A, A, A,
                                            None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_rmsnorm_quantize_act(A, 1, 1, 96, 96, None, 0, 1e-5, A, A, A, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_rmsnorm_quantize_act(A, 1, 1, 64, 64, A + 8, 0, 1e-5, A, A, A,
                                            None) == bl.BL_ERR_ALIGN
    P = ctypes.c_void_p * 1
    I = ctypes.c_int64 * 1
    pk, sc, ys = P(A), P(A), P(A)
    assert L.bitlinear_rmsnorm_gemv_fused_multi(1, pk, sc, I(64), 256, None, 1, None, 0, 1e-5, ys, 1,
                                                I(64), None, 0, None) == bl.BL_ERR_NULL
    assert L.bitlinear_rmsnorm_gemv_fused_multi(0, pk, sc, I(64), 256, A, 1, None, 0, 1e-5, ys, 1,
                                                I(64), None, 0, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_rmsnorm_gemv_fused_multi(1, pk, sc, I(64), 256, A, 1, None, 0, -2.0, ys, 1,
                                                I(64), None, 0, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_rmsnorm_gemv_fused_multi(1, pk, sc, I(64), 256, A, 1, None, 0, 1e-5, ys, 1,
                                                I(64), None, 4, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_rmsnorm_gemv_fused_multi(1, pk, sc, I(64), 256, A + 4, 1, None, 0, 1e-5, ys,
                                                1, I(64), None, 0, None) == bl.BL_ERR_ALIGN


def test_bitplane_sizes_and_argument_errors(bl):
    A = 0x7f0000000000
    L = bl.lib
    assert L.bitlinear_bitplane_bytes(28672, 8192) == 28672 * 128 * 16
    assert L.bitlinear_bitplane_bytes(8, 96) == 0
    assert L.bitlinear_bitplane_pack(None, 8, 64, A, None) == bl.BL_ERR_NULL
    assert L.bitlinear_bitplane_pack(A, 8, 65600, A, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_bitplane_pack(A + 8, 8, 64, A, None) == bl.BL_ERR_ALIGN
    assert L.bitlinear_bitplane_gemv(A, A, 8, 64, None, 1, A, 1, None, None) == bl.BL_ERR_NULL
    assert L.bitlinear_bitplane_gemv(A, A, 8, 64, A, 3, A, 1, None, None) == bl.BL_ERR_DTYPE
    assert L.bitlinear_bitplane_gemv(A, A, 8, 131072, A, 1, A, 1, None, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_bitplane_gemv(A, A, 8, 64, A + 2, 1, A, 1, None, None) == bl.BL_ERR_ALIGN


def test_lut_gemv_argument_errors(bl):
    A = 0x7f0000000000
    L = bl.lib
    assert L.bitlinear_lut_gemv(A, A, 8, 64, None, A, A, 1, None, None) == bl.BL_ERR_NULL
    assert L.bitlinear_lut_gemv(A, A, 8, 64, A, A, A, 5, None, None) == bl.BL_ERR_DTYPE
    assert L.bitlinear_lut_gemv(A, A, 8, 12352, A, A, A, 1, None, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_lut_gemv(A, A, 8, 64, A, A + 2, A, 1, None, None) == bl.BL_ERR_ALIGN


def test_chain_step_struct_matches_the_header(bl, tmp_path):
    """The binding's ctypes mirror of bitlinear_chain_step has the C layout."""
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    fields = [f[0] for f in bl.ChainStepC._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "bitlinear.h"\nint main(void){'
                   'printf("%zu", sizeof(bitlinear_chain_step));'
                   + "".join(f'printf(" %zu", offsetof(bitlinear_chain_step, {f}));' for f in fields)
                   + "return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    want = [ctypes.sizeof(bl.ChainStepC)] + [getattr(bl.ChainStepC, f).offset for f in fields]
    assert got == want


def test_chain_argument_errors(bl):
    L = bl.lib
    assert L.bitlinear_chain_plan_bytes(0) == 0
    assert L.bitlinear_chain_plan_bytes(4097) == 0
    assert L.bitlinear_chain_plan_bytes(120) > 120 * ctypes.sizeof(bl.ChainStepC)
    A = 0x7f0000000000
    st = (bl.ChainStepC * 1)()
    st[0].count = 1
    st[0].packed[0] = A
    st[0].w_scale[0] = A
    st[0].N[0] = 64
    st[0].y[0] = A
    st[0].K = 2560
    st[0].x = A
    st[0].xt = st[0].yt = 1
    nb = L.bitlinear_chain_plan_bytes(1)
    assert L.bitlinear_chain_plan(1, st, None, nb, None) == bl.BL_ERR_NULL
    assert L.bitlinear_chain_plan(0, st, A, nb, None) == bl.BL_ERR_SHAPE
    st[0].K = 2304 + 64     # not a multiple of 256
    assert L.bitlinear_chain_plan(1, st, A, nb, None) == bl.BL_ERR_SHAPE
    st[0].K = 32768         # above the chain's 16384
    assert L.bitlinear_chain_plan(1, st, A, nb, None) == bl.BL_ERR_SHAPE
    st[0].K = 2560
    st[0].eps = -1.0
    assert L.bitlinear_chain_plan(1, st, A, nb, None) == bl.BL_ERR_SHAPE
    st[0].eps = 1e-5
    st[0].xt = 9
    assert L.bitlinear_chain_plan(1, st, A, nb, None) == bl.BL_ERR_DTYPE
    st[0].xt = 1
    assert L.bitlinear_chain_plan(1, st, A, nb - 1, None) == bl.BL_ERR_WORKSPACE
    assert L.bitlinear_chain_plan(1, st, A + 8, nb, None) == bl.BL_ERR_ALIGN
    assert L.bitlinear_chain_run(None, 1, None) == bl.BL_ERR_NULL
    assert L.bitlinear_chain_run(A, 0, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_chain_run_timeout_test(A, 1, 1000000, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_chain_run_timeout_test(A, 2, 10, None) == bl.BL_ERR_SHAPE


def test_decoder_entry_argument_errors(bl):
    A = 0x7f0000000000
    L = bl.lib
    P = ctypes.c_void_p * 1
    I = ctypes.c_int64 * 1
    pk, sc, ys = P(A), P(A), P(A)
    f = L.bitlinear_decode_linear
    assert f(1, pk, sc, I(64), 256, 2, A, 1, None, None, 0, 1e-5, ys, 1, I(64), None, None, 0, None) == bl.BL_ERR_NULL
    assert f(1, pk, sc, I(64), 256, 7, A, 1, None, None, 0, 1e-5, ys, 1, I(64), None, None, 0, None) == bl.BL_ERR_SHAPE
    assert f(1, pk, sc, I(64), 256, 2, A, 0, A, None, 0, 1e-5, ys, 1, I(64), None, None, 0, None) == bl.BL_ERR_DTYPE
    assert f(1, pk, sc, I(64), 256, 0, A, 1, None, None, 0, 1e-5, ys, 0, I(64), P(A), None, 0, None) == bl.BL_ERR_DTYPE
    assert f(1, pk, sc, I(64), 256, 1, A, 1, None, None, 0, -1.0, ys, 1, I(64), None, None, 0, None) == bl.BL_ERR_SHAPE
    g = L.bitlinear_attention_decode
    nb = L.bitlinear_attention_workspace_bytes(20, 5, 64)
    assert nb > 20 * 64 * 4 and L.bitlinear_attention_workspace_bytes(20, 6, 64) == 0
    assert L.bitlinear_attention_workspace_bytes(40, 2, 64) == 0      # 20 query heads per kv head
    assert g(None, A, A, A, A, A, 20, 5, 128, 64, 1e4, None, A, A, nb, 0, None) == bl.BL_ERR_NULL
    assert g(A, A, A, A, A, A, 20, 5, 64, 64, 1e4, None, A, A, nb, 0, None) == bl.BL_ERR_SHAPE
    assert g(A, A, A, A, A, A, 20, 6, 128, 64, 1e4, None, A, A, nb, 0, None) == bl.BL_ERR_SHAPE
    assert g(A, A, A, A, A, A, 20, 5, 128, 40000, 1e4, None, A, A, nb, 0, None) == bl.BL_ERR_SHAPE
    assert g(A + 8, A, A, A, A, A, 20, 5, 128, 64, 1e4, None, A, A, nb, 0, None) == bl.BL_ERR_ALIGN
    assert g(A, A, A, A, A, A, 20, 5, 128, 64, 1e4, None, A, A + 8, nb, 0, None) == bl.BL_ERR_ALIGN
    assert L.bitlinear_position_advance(None, None) == bl.BL_ERR_NULL
    assert L.bitlinear_position_advance(A + 2, None) == bl.BL_ERR_ALIGN


def test_rope_table_argument_errors(bl):
    A = 0x7f0000000000
    L = bl.lib
    assert L.bitlinear_rope_table(128, 64, 1e4, None, None) == bl.BL_ERR_NULL
    assert L.bitlinear_rope_table(64, 64, 1e4, A, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_rope_table(128, 0, 1e4, A, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_rope_table(128, 64, 0.5, A, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_rope_table(128, 64, 1e4, A + 4, None) == bl.BL_ERR_ALIGN


def test_gemv_plan_argument_errors(bl):
    """bitlinear_gemv_plan checks its arguments before it asks for a device."""
    import torch
    L = bl.lib
    N = (ctypes.c_int64 * 2)(2560, 640)
    k, c = ctypes.c_int(0), ctypes.c_int(0)
    kp, cp = ctypes.byref(k), ctypes.byref(c)
    assert L.bitlinear_gemv_plan(2, None, 2560, 4, 1, 1, 0, kp, cp) == bl.BL_ERR_NULL
    assert L.bitlinear_gemv_plan(2, N, 2560, 4, 1, 1, 0, None, cp) == bl.BL_ERR_NULL
    assert L.bitlinear_gemv_plan(0, N, 2560, 4, 1, 1, 0, kp, cp) == bl.BL_ERR_SHAPE
    assert L.bitlinear_gemv_plan(2, N, 2560, 17, 1, 1, 0, kp, cp) == bl.BL_ERR_SHAPE
    assert L.bitlinear_gemv_plan(2, N, 2560, 4, 1, 1, 8, kp, cp) == bl.BL_ERR_SHAPE
    assert L.bitlinear_gemv_plan(2, N, 2560, 4, 9, 1, 0, kp, cp) == bl.BL_ERR_DTYPE
    if not torch.cuda.is_available():
        st = L.bitlinear_gemv_plan(2, N, 2560, 4, 1, 1, 0, kp, cp)
        assert st in (bl.BL_ERR_CUDA, bl.BL_ERR_UNSUPPORTED)


def test_probe_argument_errors(bl):
    """The tensor-core probes check their shapes before any CUDA call."""
    A = 0x7f0000000000
    L = bl.lib
    assert L.bitlinear_probe_mma_i8(100, None, 1, None) == bl.BL_ERR_NULL
    assert L.bitlinear_probe_mma_i8(0, A, 1, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_probe_mma_i8_issue(64, 1, 100, A, 1, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_probe_mma_i8_issue(32, 3, 100, A, 1, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_probe_mma_i8_issue(128, 4, 100, A, 1, None) == bl.BL_ERR_SHAPE
    assert L.bitlinear_probe_mma_i8_issue(32, 4, 100, A + 4, 1, None) == bl.BL_ERR_ALIGN


def test_binding_constants_match_the_header(bl):
    """The binding's launch flags and kernel ids are the header's."""
    text = open(os.path.join(ROOT, "include", "bitlinear.h")).read()
    defs = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define\s+(BL_\w+)\s+(\d+)u?\b", text)}
    for name in ("BL_FLAG_PDL", "BL_FLAG_SMALL_BATCH_DP4A", "BL_FLAG_SMALL_BATCH_TENSOR"):
        assert getattr(bl, name) == defs[name], name
    kernels = {v: k for k, v in bl.GEMV_KERNELS.items()}
    assert kernels["stream"] == defs["BL_GEMV_KERNEL_STREAM"]
    assert kernels["tensor"] == defs["BL_GEMV_KERNEL_TENSOR"]
    assert kernels["stream_mt"] == defs["BL_GEMV_KERNEL_STREAM_MT"]
    assert kernels["dp4a"] == defs["BL_GEMV_KERNEL_DP4A"]
    assert bl.BL_ACT_PLAIN == defs["BL_ACT_PLAIN"] and bl.BL_ACT_RMSNORM == defs["BL_ACT_RMSNORM"]
    assert bl.BL_ACT_RELU2_GATE == defs["BL_ACT_RELU2_GATE"]


_C_HOST = r"""
#include <stdio.h>
#include <stdint.h>
#include "bitlinear.h"

int main(void)
{
    /* sizes and strings need no device */
    printf("%zu %zu %s\n", bitlinear_packed_bytes(13, 256), bitlinear_packed_bytes(8, 100),
           bitlinear_status_string(BL_ERR_SHAPE));
    /* argument errors come back before any CUDA call */
    uintptr_t a = (uintptr_t)0x7f0000000000ull;
    const uint8_t *packed = (const uint8_t *)a;
    const float *scale = (const float *)a;
    const int8_t *q = (const int8_t *)a;
    const float *d = (const float *)a;
    const int32_t *r = (const int32_t *)a;
    void *y = (void *)a;
    int s1 = bitlinear_gemv(packed, scale, 256, 256, NULL, d, r, 1, y, BL_BF16, 256, NULL, NULL);
    int s2 = bitlinear_gemv(packed, scale, 256, 100, q, d, r, 1, y, BL_BF16, 256, NULL, NULL);
    int s3 = bitlinear_gemv(packed, scale, 256, 256, q, d, r, 1, y, 7, 256, NULL, NULL);
    printf("%d %d %d\n", s1, s2, s3);
    return 0;
}
"""


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c11"), ("g++", "-std=c++17")])
def test_plain_c_host_links_and_calls_the_library(bl, tmp_path, compiler, std):
    """A C (and a C++) program with no Python or torch includes the header
    under strict warnings, links libbitlinear.so and gets the documented
    sizes, strings and argument errors."""
    import shutil
    import subprocess
    if not shutil.which(compiler):
        pytest.skip("no compiler")
    src = tmp_path / ("host.c" if compiler == "gcc" else "host.cpp")
    src.write_text(_C_HOST)
    exe = tmp_path / "host"
    libdir = os.path.dirname(bl.LIB_PATH)
    subprocess.run([compiler, std, "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-lbitlinear", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    first = out[0].split(" ", 2)
    assert int(first[0]) == oracle.packed_bytes(13, 256) and int(first[1]) == 0
    assert first[2].startswith("BL_ERR_SHAPE")
    assert [int(v) for v in out[1].split()] == [bl.BL_ERR_NULL, bl.BL_ERR_SHAPE, bl.BL_ERR_DTYPE]
