"""The oracle's pins catch plausible mistakes: each mutant below plants one mistake in a copy
of oracle/nvfp4_oracle.c (a flipped tie rule, a dropped sign or term, a wrong constant,
index or stride, a transposed layout, an inexact division), and the oracle's pin tests must
fail against that copy. Everything runs on the CPU in a scratch directory; the repository's
oracle is never modified.

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

MUTANTS = [
    ("e2m1 ties to the odd code",
     "      if (d < best_d || (d == best_d && (c & 1) == 0)) {",
     "      if (d < best_d || (d == best_d && (c & 1) == 1)) {"),
    ("e4m3 ties to the odd code",
     "\n    if (d < best_d || (d == best_d && (c & 1) == 0)) {",
     "\n    if (d < best_d || (d == best_d && (c & 1) == 1)) {"),
    ("e2m1 sign dropped", "return (sign << 3) | best;", "return best;"),
    ("e4m3 subnormal step", "mag = ldexp((double)m, -9);", "mag = ldexp((double)m, -10);"),
    ("global scale 448 / amax", "float g = 2688.0f / amax;", "float g = 448.0f / amax;"),
    ("block scale without / 6", "float s = (amax_b / 6.0f) * g;", "float s = amax_b * g;"),
    ("reciprocal instead of division",
     "float r = (s_dec == 0.0f) ? 0.0f : g / s_dec;",
     "float r = (s_dec == 0.0f) ? 0.0f : g * (1.0f / s_dec);"),
    ("nibbles swapped",
     "q[j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));",
     "q[j] = (uint8_t)((codes[2 * j + 1] & 0xF) | ((codes[2 * j] & 0xF) << 4));"),
    ("128x4 strides swapped",
     "return atom * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4);",
     "return atom * 512 + (r % 32) * 4 + ((r / 32) % 4) * 16 + (c % 4);"),
    ("8x4 atom transposed",
     "return atom * 32 + (r % 8) * 4 + (c % 4);",
     "return atom * 32 + (r % 8) + (c % 4) * 8;"),
    ("GEMM weight scale block index",
     "orc_e4m3_value(sw[n * (K / 16) + k / 16]) /\n                    (double)gw;",
     "orc_e4m3_value(sw[n * (K / 16) + k / 32]) /\n                    (double)gw;"),
    ("GEMM weight global scale dropped",
     "orc_e4m3_value(sw[n * (K / 16) + k / 16]) /\n                    (double)gw;",
     "orc_e4m3_value(sw[n * (K / 16) + k / 16]);"),
    ("exp Taylor term dropped", "for (int n = 6; n >= 0; --n)", "for (int n = 5; n >= 0; --n)"),
    ("exp ln2_lo dropped", "f = fmaf(-k, ORC_LN2_LO, f);", ""),
]


def _run_mutant(base, index, old, new, src):
    work = os.path.join(base, f"m{index}")
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(work, "oracle"),
                    ignore=shutil.ignore_patterns("_liboracle*", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(work, "tests"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    with open(os.path.join(work, "oracle", "nvfp4_oracle.c"), "w") as f:
        f.write(src.replace(old, new))
    # the copied tests put `work` first on sys.path, so `import oracle` finds the mutant
    env = dict(os.environ, PYTHONPATH=work + os.pathsep + ROOT)
    out = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          "-m", "not gpu", *PIN_TESTS], cwd=work, env=env, capture_output=True,
                         text=True, timeout=900)
    return out.returncode, out.stdout[-2000:]


def test_pins_catch_every_mutant(tmp_path):
    with open(os.path.join(ROOT, "oracle", "nvfp4_oracle.c")) as f:
        src = f.read()
    for name, old, _ in MUTANTS:
        assert src.count(old) == 1, f"mutation site not unique or missing: {name}"
    with ThreadPoolExecutor(max_workers=4) as ex:
        results = list(ex.map(lambda im: _run_mutant(str(tmp_path), im[0], im[1][1], im[1][2], src),
                              enumerate(MUTANTS)))
    survivors = []
    for (name, _, _), (rc, tail) in zip(MUTANTS, results):
        # 1 = some test failed (caught); 0 = every pin passed (survived); other codes = broken run
        assert rc in (0, 1), f"{name}: pytest exit {rc}\n{tail}"
        if rc == 0:
            survivors.append(name)
    assert not survivors, f"mutants no pin caught: {survivors}"
