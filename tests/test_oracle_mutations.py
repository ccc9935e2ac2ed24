"""The oracle's pins catch plausible mistakes (no GPU).

Each case plants ONE mistake -- a dropped term, a wrong sign or index, a
transposed operand, another rounding rule, a step composed in the wrong
order -- in a copy of the oracle: of its C source (built with the oracle's
own compiler flags and selected through BITLINEAR_ORACLE_LIB) or of its
Python module (loaded as ``oracle`` in place of the real one).  The pins
(tests/test_oracle_pins.py) then run in a child process and must fail.
Control copies of the unchanged C source and module must pass them, so a
failure is the planted mistake's doing.  Everything is planted in copies
under a temporary directory; the oracle's own files are never touched.
"""
import concurrent.futures as cf
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "bitlinear_oracle.c")
PY = os.path.join(ROOT, "oracle", "__init__.py")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (what the mistake is, exact text in the source, replacement)
MUTATIONS = [
    # weight scale (mean |W| in fp64, floor 1e-5)
    ("weight scale: |w| dropped", "row += fabs((double)W[n * K + k]);",
     "row += (double)W[n * K + k];"),
    ("weight scale: sum over N instead of N*K", "(float)(S / (double)(N * K))",
     "(float)(S / (double)N)"),
    ("weight scale: no 1e-5 floor", "return gamma > ORACLE_EPS ? gamma : ORACLE_EPS;",
     "return gamma;"),
    # ternary round-clip
    ("codes: ties away from zero", "float t = rintf(r);", "float t = roundf(r);"),
    ("codes: sign flipped", "            c = 1;\n        else if (t <= -1.0f)\n            c = -1;",
     "            c = -1;\n        else if (t <= -1.0f)\n            c = 1;"),
    # TL layout
    ("layout: word and byte indices swapped", "* 16 + w * 4 + j;", "* 16 + j * 4 + w;"),
    ("layout: 2-bit field from k % 4", "return (int)(2 * ((k % 16) / 4));",
     "return (int)(2 * (k % 4));"),
    ("layout: codes stored in two's complement", "unsigned s = (unsigned)(code + 1);",
     "unsigned s = (unsigned)(code & 3);"),
    ("layout: pad rows hold code -1", "int code = n < N ? codes[n * K + k] : 0;",
     "int code = n < N ? codes[n * K + k] : -1;"),
    # activation quantisation
    ("quant: ties away from zero", "float t = rintf(v);", "float t = roundf(v);"),
    ("quant: Qb = 128", "#define ORACLE_QB 127.0f", "#define ORACLE_QB 128.0f"),
    ("quant: max x instead of max |x|", "float a = fabsf(xm[k]);", "float a = xm[k];"),
    ("quant: inverted dequantisation scale", "d[m] = a_eff / ORACLE_QB;",
     "d[m] = ORACLE_QB / a_eff;"),
    ("quant: row sum of |q|", "r += qi;", "r += qi < 0 ? -qi : qi;"),
    # product and rescale
    ("product: -1 codes add", "s -= qm[k];", "s += qm[k];"),
    ("product: output transposed", "acc[m * N + n] = (int32_t)s;", "acc[n * M + m] = (int32_t)s;"),
    ("rescale: first token's scale for all", "float t = a * d[m];", "float t = a * d[0];"),
    ("rescale: weight scale dropped", "y[m * N + n] = t * gamma_eff;", "y[m * N + n] = t;"),
    ("bf16: ties away from zero", "u += 0x7fffu + lsb;", "u += 0x8000u;"),
    # binary variant
    ("binary: zero counted negative", "bit = v[r * K + k] < 0.0f ? 1u : 0u;",
     "bit = v[r * K + k] <= 0.0f ? 1u : 0u;"),
    ("binary: XOR instead of XNOR", "pc += popcount64_plain(~(Wb[n * words + w] ^ xb[w]));",
     "pc += popcount64_plain(Wb[n * words + w] ^ xb[w]);"),
    ("binary: pad bits counted", "acc[n] = (int32_t)(2 * pc - K);",
     "acc[n] = (int32_t)(2 * pc - 64 * words);"),
    ("binary: activation scale dropped", "float s = s_w * s_x;", "float s = s_w;"),
    # bit-planes
    ("bit-planes: sign bits on positive weights", "if (c < 0)\n                    s |=",
     "if (c > 0)\n                    s |="),
    ("bit-planes: second popcount added", "dot -= popcount64_plain(m & (s ^ xb[w]));",
     "dot += popcount64_plain(m & (s ^ xb[w]));"),
    # RMSNorm
    ("rmsnorm: epsilon dropped", "float den = sqrtf(ms + eps);", "float den = sqrtf(ms);"),
    ("rmsnorm: sum instead of mean", "float ms = (float)(S / (double)K);", "float ms = (float)S;"),
    ("rmsnorm: gain divides", "h[m * K + k] = gain ? t * gain[k] : t;",
     "h[m * K + k] = gain ? t / gain[k] : t;"),
    # decoder-layer pieces
    ("rope: rotation sign", "out[h * D + 2 * i] = ac - bs;", "out[h * D + 2 * i] = ac + bs;"),
    ("rope: angle schedule", "pow(base, -(double)(2 * i) / (double)D)",
     "pow(base, -(double)i / (double)D)"),
    ("attention: kv head by modulo", "int64_t kv = h / (H / Hkv);", "int64_t kv = h % Hkv;"),
    ("attention: 1/sqrt(D) dropped", "float scale = (float)(1.0 / sqrt((double)D));",
     "float scale = 1.0f;"),
    ("attention: softmax not normalised", "out[h * D + d] = (float)(num / S);",
     "out[h * D + d] = (float)num;"),
    ("gate: ReLU not squared", "float rr = r * r;", "float rr = r;"),
    ("gate: no ReLU", "float r = g[i] > 0.0f ? g[i] : 0.0f;", "float r = g[i];"),
    ("residual: stream dropped", "out[i] = h[i] + y[i];", "out[i] = y[i];"),
]

# mistakes in the Python module: the composed paths (binary and bit-plane
# GEMVs, a decoder layer around its BitLinears)
PY_MUTATIONS = [
    ("binary: x pad bits 0", "xb = binary_signs(x, pad_bit=1)", "xb = binary_signs(x, pad_bit=0)"),
    ("binary: weight scale from x", "s_w = absmax(W)", "s_w = absmax(x)"),
    ("bit-planes: gamma dropped", '"y": binary_rescale(acc, gamma_eff, s_x)}',
     '"y": binary_rescale(acc, 1.0, s_x)}'),
    ("RMSNorm + quantiser: the norm skipped", "return quantize_act(rmsnorm(x, gain, eps))",
     "return quantize_act(x)"),
    ("layer: attention misses the current position",
     "attention_decode(q_rot, cache_k, cache_v, H, Hkv, D, pos + 1)",
     "attention_decode(q_rot, cache_k, cache_v, H, Hkv, D, pos)"),
    ("layer: attention normalised with the FFN gain",
     'layer["q"][0], layer["g_attn"], eps))\n'
     '    k = bf16_round(_linear32(h, layer["k"][1], layer["k"][0], layer["g_attn"], eps))\n'
     '    v = bf16_round(_linear32(h, layer["v"][1], layer["v"][0], layer["g_attn"], eps))',
     'layer["q"][0], layer["g_ffn"], eps))\n'
     '    k = bf16_round(_linear32(h, layer["k"][1], layer["k"][0], layer["g_ffn"], eps))\n'
     '    v = bf16_round(_linear32(h, layer["v"][1], layer["v"][0], layer["g_ffn"], eps))'),
    ("layer: FFN normalised with the attention gain",
     'layer["gate"][0], layer["g_ffn"], eps))\n'
     '    up = bf16_round(_linear32(h1, layer["up"][1], layer["up"][0], layer["g_ffn"], eps))',
     'layer["gate"][0], layer["g_attn"], eps))\n'
     '    up = bf16_round(_linear32(h1, layer["up"][1], layer["up"][0], layer["g_attn"], eps))'),
    ("layer: RMSNorm gain dropped", "x32 = rmsnorm(x32, gain, eps)", "x32 = rmsnorm(x32, None, eps)"),
    ("layer: keys not rotated", "k_rot = bf16_round(rope(k, Hkv, D, pos, base))", "k_rot = k"),
    ("layer: keys rotated for the next position", "k_rot = bf16_round(rope(k, Hkv, D, pos, base))",
     "k_rot = bf16_round(rope(k, Hkv, D, pos + 1, base))"),
    ("layer: values rotated", "cache_v[:, pos, :] = v.reshape(Hkv, D)",
     "cache_v[:, pos, :] = bf16_round(rope(v, Hkv, D, pos, base)).reshape(Hkv, D)"),
    ("layer: values cached from the keys", "cache_v[:, pos, :] = v.reshape(Hkv, D)",
     "cache_v[:, pos, :] = k.reshape(Hkv, D)"),
    ("layer: gate and up exchanged", "m = relu2_gate(gate, up)", "m = relu2_gate(up, gate)"),
    ("layer: FFN residual skips the attention output", "return bf16_round(residual_add(h1, y_d))",
     "return bf16_round(residual_add(h, y_d))"),
]


def _cflags():
    import oracle
    return list(oracle._CFLAGS)


def _build(src_text: str, path: str):
    c = path + ".c"
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", *_cflags(), "-o", path, c, "-lm"], check=True,
                   capture_output=True)


def _run_pins(lib: str, module: str | None = None) -> subprocess.CompletedProcess:
    """The pins in a child process, with the oracle on the C library `lib`
    and, when given, the Python module file `module` loaded as ``oracle``."""
    env = dict(os.environ, BITLINEAR_ORACLE_LIB=lib, OMP_NUM_THREADS="1")
    args = ["-x", "-q", "-p", "no:cacheprovider", PINS]
    if module is None:
        cmd = [sys.executable, "-m", "pytest", *args]
    else:
        boot = ("import importlib.util, sys\n"
                f"spec = importlib.util.spec_from_file_location('oracle', {module!r}, "
                f"submodule_search_locations=[{os.path.dirname(module)!r}])\n"
                "mod = importlib.util.module_from_spec(spec)\n"
                "sys.modules['oracle'] = mod\n"
                "try:\n"
                "    spec.loader.exec_module(mod)\n"
                "except Exception:\n"
                "    sys.exit(97)\n"
                "import pytest\n"
                f"sys.exit(pytest.main({args!r}))\n")
        cmd = [sys.executable, "-c", boot]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.fixture(scope="module")
def module_source():
    with open(PY) as f:
        return f.read()


def test_every_mutation_names_one_place_in_the_source(source, module_source):
    for muts, text in ((MUTATIONS, source), (PY_MUTATIONS, module_source)):
        for what, old, new in muts:
            assert text.count(old) == 1, what
            assert old != new, what


def _module(text: str, path) -> str:
    path.mkdir()
    f = path / "__init__.py"
    f.write_text(text)
    return str(f)


def test_pins_fail_on_every_planted_mistake(source, module_source, tmp_path):
    control = str(tmp_path / "control.so")
    _build(source, control)
    jobs = [("control", control, None),
            ("control module", control, _module(module_source, tmp_path / "control_py"))]
    for i, (what, old, new) in enumerate(MUTATIONS):
        lib = str(tmp_path / f"mut{i}.so")
        _build(source.replace(old, new), lib)
        jobs.append((what, lib, None))
    for i, (what, old, new) in enumerate(PY_MUTATIONS):
        jobs.append((what, control, _module(module_source.replace(old, new), tmp_path / f"py{i}")))
    workers = max(1, min(8, os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(workers) as ex:
        results = dict(zip([j[0] for j in jobs], ex.map(lambda j: _run_pins(j[1], j[2]), jobs)))
    for name in ("control", "control module"):
        ctl = results.pop(name)
        assert ctl.returncode == 0, f"{name}: the unchanged oracle fails its pins:\n" + \
            ctl.stdout[-2000:] + ctl.stderr[-2000:]
    # exit code 1: the run completed and a pin failed (not a crash, a
    # collection error or a module that does not load)
    survived = {w: r.returncode for w, r in results.items() if r.returncode != 1}
    assert not survived, f"mistakes the pins do not catch (pytest exit code): {survived}"
