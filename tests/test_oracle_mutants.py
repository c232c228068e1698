"""Mutation tests of the oracle's pins.

The oracle source carries numbered plausible mistakes behind ORC_MUTANT (see
the header of oracle/mxfp4_oracle.c).  Each one is built into its own library
and the oracle pin suite is run against it in a subprocess: every mutant must
make at least one pin fail.  A mutant that survives would mean the pins could
not tell that mistake from the definition on the pages.
"""
import concurrent.futures
import os
import re
import subprocess
import sys

import pytest

from oracle import build as oracle_build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

MUTANTS = {
    1: "RNE ties go away from zero instead of to the even code",
    2: "scale exponent floor(log2 amax) - 1 instead of - 2",
    3: "SR threshold f * 2^31 instead of f * 2^32",
    4: "nibbles packed high-first",
    5: "RHT sign word drawn from the wrong counter word",
    6: "negative zero stored with a + sign",
    7: "GEMM block factor 2^(ea - eb) instead of 2^(ea + eb)",
    8: "2D transposed copy misplaces rows",
    9: "NaN in a block not turned into the NaN scale",
    10: "Philox with 9 rounds instead of 10",
    11: "RHT without the 1/sqrt(d) normalisation",
    12: "SR ignores the element offset",
    13: "amax over signed values instead of magnitudes",
    14: "dequantize ignores the block scale",
    15: "E8M0 decoded with bias 128",
    16: "butterfly stores (b - a) instead of (a - b)",
    17: "column layout draws SR words by input index instead of output index",
    19: "GEMM pairs element k of A with element k^1 of B",
    20: "dequantize skips the inverse RHT",
    21: "round-up scale compares against 5 * 2^e instead of 6 * 2^e",
    22: "3/4 pre-scale also applied to the amax that sets the exponent",
    23: "NVFP4 tensor scale amax / (6 * 256) instead of / (6 * 448)",
    24: "E4M3 rounding ties to the odd code",
    25: "NVFP4 GEMM drops the per-tensor scales",
    26: "NVFP4 element divisor without the tensor scale",
    27: "bf16 output rounding ties away from zero",
    28: "bf16 output truncated instead of rounded",
    29: "2D dequantize reads the tile scale at the 1D row index",
    30: "1D-column dequantize swaps the two elements of each byte",
}

PIN_FILES = ["test_oracle_format.py", "test_oracle_gemm.py", "test_oracle_quantize.py", "test_oracle_rht.py",
             "test_oracle_sr.py", "test_oracle_scale_rules.py", "test_oracle_nvfp4.py", "test_oracle_philox.py",
             "test_oracle_bf16.py"]


@pytest.fixture(scope="module")
def workdir(tmp_path_factory):
    d = tmp_path_factory.mktemp("mutants")
    sys.path.insert(0, HERE)
    from test_oracle_philox import build_torch_philox
    return str(d), build_torch_philox(str(d))


def _run_pins(lib: str, philox_exe: str):
    env = dict(os.environ, MXFP4_ORACLE_LIB=lib, MXFP4_TORCH_PHILOX=philox_exe, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-rf", "-p", "no:cacheprovider", "-m", "not gpu",
           *[os.path.join(HERE, f) for f in PIN_FILES]]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    failed = re.findall(r"^FAILED (\S+)", r.stdout, re.M)
    return r.returncode, failed, r.stdout[-2000:]


def test_every_planted_mistake_fails_a_pin(workdir):
    d, philox_exe = workdir

    def one(k):
        lib = oracle_build.build(mutant=k, out=os.path.join(d, f"liboracle_mutant{k}.so"))
        return k, *_run_pins(lib, philox_exe)

    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(one, sorted(MUTANTS)))
    survivors = []
    for k, rc, failed, tail in results:
        # exit code 1 = some test failed; anything else (errors, no tests) is not a kill
        if rc != 1 or not failed:
            survivors.append(f"mutant {k} ({MUTANTS[k]}): exit {rc}\n{tail}")
    assert not survivors, "\n".join(survivors)
