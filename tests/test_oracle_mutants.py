"""The oracle's pins catch plausible mistakes: each mutant below plants one mistake in a copy
of the oracle (oracle/nvfp4_oracle.c or oracle/__init__.py: a flipped tie rule, a dropped
sign, term or scale, a wrong constant, index, stride or operand order, a transposed layout, an
inexact division, a skipped rounding), and the oracle's pin tests must fail against that copy.
Everything runs on the CPU in a scratch directory; the repository's oracle is never modified.

Not listed: the form of the silu division (v / (1 + e) against v * (1 / (1 + e))). That is a
reading of the pages; no value outside the oracle fixes it."""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_TESTS = ["tests/test_oracle_codecs.py", "tests/test_oracle_quantize.py",
             "tests/test_oracle_layout_gemm.py"]

C, PY = "nvfp4_oracle.c", "__init__.py"

MUTANTS = [  # (what, file, original text, planted text)
    ("e2m1 ties to the odd code", C,
     "      if (d < best_d || (d == best_d && (c & 1) == 0)) {",
     "      if (d < best_d || (d == best_d && (c & 1) == 1)) {"),
    ("e4m3 ties to the odd code", C,
     "\n    if (d < best_d || (d == best_d && (c & 1) == 0)) {",
     "\n    if (d < best_d || (d == best_d && (c & 1) == 1)) {"),
    ("e2m1 sign dropped", C, "return (sign << 3) | best;", "return best;"),
    ("e4m3 subnormal step", C, "mag = ldexp((double)m, -9);", "mag = ldexp((double)m, -10);"),
    ("global scale 448 / amax", C, "float g = 2688.0f / amax;", "float g = 448.0f / amax;"),
    ("block scale without / 6", C, "float s = (amax_b / 6.0f) * g;", "float s = amax_b * g;"),
    ("reciprocal instead of division", C,
     "float r = (s_dec == 0.0f) ? 0.0f : g / s_dec;",
     "float r = (s_dec == 0.0f) ? 0.0f : g * (1.0f / s_dec);"),
    ("nibbles swapped", C,
     "q[j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));",
     "q[j] = (uint8_t)((codes[2 * j + 1] & 0xF) | ((codes[2 * j] & 0xF) << 4));"),
    ("128x4 strides swapped", C,
     "return atom * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4);",
     "return atom * 512 + (r % 32) * 4 + ((r / 32) % 4) * 16 + (c % 4);"),
    ("8x4 atom transposed", C,
     "return atom * 32 + (r % 8) * 4 + (c % 4);",
     "return atom * 32 + (r % 8) + (c % 4) * 8;"),
    ("GEMM weight scale block index", C,
     "orc_e4m3_value(sw[n * (K / 16) + k / 16]) /\n                    (double)gw;",
     "orc_e4m3_value(sw[n * (K / 16) + k / 32]) /\n                    (double)gw;"),
    ("GEMM weight global scale dropped", C,
     "orc_e4m3_value(sw[n * (K / 16) + k / 16]) /\n                    (double)gw;",
     "orc_e4m3_value(sw[n * (K / 16) + k / 16]);"),
    ("exp Taylor term dropped", C, "for (int n = 6; n >= 0; --n)", "for (int n = 5; n >= 0; --n)"),
    ("exp ln2_lo dropped", C, "f = fmaf(-k, ORC_LN2_LO, f);", ""),
    ("silu of +v", C, "float orc_silu(float v) { return v / (1.0f + orc_exp(-v)); }",
     "float orc_silu(float v) { return v / (1.0f + orc_exp(v)); }"),
    ("fused SwiGLU quantize: gate and up swapped", C,
     "        yb[i] = orc_swiglu_elem(load_elem(x, dtype, r * ldx + h),\n"
     "                                load_elem(x, dtype, r * ldx + H + h));",
     "        yb[i] = orc_swiglu_elem(load_elem(x, dtype, r * ldx + H + h),\n"
     "                                load_elem(x, dtype, r * ldx + h));"),
    ("SwiGLU: gate and up swapped", C,
     "      y[r * H + h] =\n"
     "          orc_swiglu_elem(load_elem(x, dtype, r * ldx + h), load_elem(x, dtype, r * ldx + H + h));",
     "      y[r * H + h] =\n"
     "          orc_swiglu_elem(load_elem(x, dtype, r * ldx + H + h), load_elem(x, dtype, r * ldx + h));"),
    ("SwiGLU + FP8: gate and up swapped", C,
     "      const float y =\n"
     "          orc_swiglu_elem(load_elem(x, dtype, r * ldx + h), load_elem(x, dtype, r * ldx + H + h));",
     "      const float y =\n"
     "          orc_swiglu_elem(load_elem(x, dtype, r * ldx + H + h), load_elem(x, dtype, r * ldx + h));"),
    ("SwiGLU + FP8: scale divides", C, "orc_e4m3_encode_signed(y * scale);",
     "orc_e4m3_encode_signed(y / scale);"),
    ("signed E4M3 drops the sign", C, "return sign | orc_e4m3_encode(fabsf(v));",
     "return orc_e4m3_encode(fabsf(v));"),
    ("per-token scale from row 0", C,
     "gr = orc_global_scale(orc_amax(x + r * ldx, dtype, 1, K, ldx));",
     "gr = orc_global_scale(orc_amax(x, dtype, 1, K, ldx));"),
    ("fp32-scale GEMM drops the weight scale", PY,
     "dw = dequantize(w_q, w_sf_lin, 1.0) * float(np.float32(w_scale))",
     "dw = dequantize(w_q, w_sf_lin, 1.0)"),
    ("fp32-scale GEMM tiles the block scales", PY,
     "da = e2m1_a * np.repeat(s32, 16, axis=1)", "da = e2m1_a * np.tile(s32, (1, 16))"),
    ("row-parallel ranks not rounded to fp16", PY,
     "parts16.append(p16.view(np.float16).astype(np.float64))", "parts16.append(p64)"),
    ("row-parallel scale shard", PY,
     "b0, b1, c0, c1 = r * ks // 2, (r + 1) * ks // 2, r * ks // 16, (r + 1) * ks // 16",
     "b0, b1, c0, c1 = r * ks // 2, (r + 1) * ks // 2, 0, ks // 16"),
]


def _source(name):
    with open(os.path.join(ROOT, "oracle", name)) as f:
        return f.read()


def _run_mutant(base, index, fname, old, new):
    work = os.path.join(base, f"m{index}")
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(work, "oracle"),
                    ignore=shutil.ignore_patterns("_liboracle*", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(work, "tests"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    with open(os.path.join(work, "oracle", fname), "w") as f:
        f.write(_source(fname).replace(old, new))
    # the copied tests put `work` first on sys.path, so `import oracle` finds the mutant
    env = dict(os.environ, PYTHONPATH=work + os.pathsep + ROOT)
    out = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          "-m", "not gpu", *PIN_TESTS], cwd=work, env=env, capture_output=True,
                         text=True, timeout=900)
    return out.returncode, out.stdout[-2000:]


def test_pins_catch_every_mutant(tmp_path):
    for name, fname, old, _ in MUTANTS:
        assert _source(fname).count(old) == 1, f"mutation site not unique or missing: {name}"
    workers = max(2, min(8, os.cpu_count() or 2))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        results = list(ex.map(lambda im: _run_mutant(str(tmp_path), im[0], *im[1][1:]),
                              enumerate(MUTANTS)))
    survivors = []
    for (name, _, _, _), (rc, tail) in zip(MUTANTS, results):
        # 1 = some test failed (caught); 0 = every pin passed (survived); other codes = broken run
        assert rc in (0, 1), f"{name}: pytest exit {rc}\n{tail}"
        if rc == 0:
            survivors.append(name)
    assert not survivors, f"mutants no pin caught: {survivors}"
