"""The oracle and the CUDA path stay independent: the product package never imports or links
the oracle, and the oracle includes none of the CUDA path's headers (CPU only)."""
import glob
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "nvfp4_block_scaled_10_b200")


def test_importing_the_package_loads_no_oracle():
    code = ("import sys; sys.path.insert(0, %r)\n"
            "import nvfp4_block_scaled_10_b200, nvfp4_block_scaled_10_b200.tp, "
            "nvfp4_block_scaled_10_b200.workloads, nvfp4_block_scaled_10_b200.build\n"
            "print('oracle' in sys.modules)") % ROOT
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip().splitlines()[-1] == "False"


def test_package_sources_do_not_reference_the_oracle():
    pattern = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b)|nvfp4_oracle|_liboracle", re.M)
    files = [f for ext in ("py", "cu", "cuh", "h") for f in glob.glob(os.path.join(PKG, "**", "*." + ext),
                                                                     recursive=True)]
    files += glob.glob(os.path.join(ROOT, "include", "*.h"))
    assert files
    for f in files:
        with open(f) as fh:
            assert not pattern.search(fh.read()), f


def test_oracle_includes_no_cuda_path_header():
    with open(os.path.join(ROOT, "oracle", "nvfp4_oracle.c")) as fh:
        includes = re.findall(r'^\s*#\s*include\s*[<"]([^>"]+)[>"]', fh.read(), re.M)
    ours = {os.path.basename(p) for p in glob.glob(os.path.join(PKG, "csrc", "*"))}
    ours |= {os.path.basename(p) for p in glob.glob(os.path.join(ROOT, "include", "*.h"))}
    assert includes and not (set(map(os.path.basename, includes)) & ours), includes


def test_bench_loads_the_oracle_only_for_its_baselines():
    """bench.py imports the oracle inside its CPU-baseline and reference-arm functions only."""
    code = ("import sys, importlib.util; sys.path.insert(0, %r)\n"
            "spec = importlib.util.spec_from_file_location('bench', %r)\n"
            "m = importlib.util.module_from_spec(spec); spec.loader.exec_module(m)\n"
            "print('oracle' in sys.modules)") % (ROOT, os.path.join(ROOT, "bench.py"))
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip().splitlines()[-1] == "False"
    with open(os.path.join(ROOT, "bench.py")) as fh:
        src = fh.read()
    users = set()
    for fn in re.finditer(r"^def (\w+)\(.*?(?=^def |\Z)", src, re.M | re.S):
        if re.search(r"^\s+import oracle\b", fn.group(0), re.M):
            users.add(fn.group(1))
    assert users and users <= {"_oracle_sample", "cpu_baseline", "_all_cores", "_oracle_rows",
                               "run_reference"}, users
