"""The quantize kernels replace two IEEE fp32 divisions by cheaper sequences that give the
same bits: fl(amax_b / 6) by a multiply and two FMA corrections, and the per-row
r = g / s_dec by a 16-entry table of fl(g / k) scaled by a power of two. These are not
checked against the oracle here (the GPU parity tests do that on real data); this test
enumerates every input the shortcuts can meet and compares them with the division itself,
in C on the CPU."""
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("shortcuts") / "exact_shortcuts")
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", exe,
                    os.path.join(HERE, "native", "exact_shortcuts.c"), "-lm"], check=True)
    return exe


def test_row_reciprocal_table_equals_division_for_every_row_scale(checker):
    out = subprocess.run([checker, "--rtab-only"], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout


def test_division_by_six_shortcut_over_all_fp32(checker):
    out = subprocess.run([checker], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout
