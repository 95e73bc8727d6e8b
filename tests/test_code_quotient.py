"""The quantisation kernels' code arithmetic against the method's definition,
exhaustively over its whole input domain (no GPU).

The kernels never divide: the code of x is rint of a one-step reciprocal
refinement of x / s (Markstein, IBM J. Res. Dev. 34(1), 1990).  The method
defines it as rint of the IEEE quotient RN(x / s) ("Issue 5 probe: int8
quantized DiT serve paths on the RTX 3090", Round two: dynamic per-token
symmetric int8 activations).  `exhaustive/code_quotient.c` compares the two
for every bf16 row maximum with s = RN(amax / 127) >= 1e-30 and every bf16
x in [0, amax] -- about 5.2e8 pairs -- and this test asserts that none
differ, while the unrefined product x * RN(1/s) does differ (so the check
can tell the two apart).
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_one_step_quotient_gives_the_ieee_codes(tmp_path):
    exe = str(tmp_path / "code_quotient")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-o", exe,
                    os.path.join(HERE, "exhaustive", "code_quotient.c"), "-lm"], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=1800).stdout
    fields = out.split()
    got = {fields[i]: int(fields[i + 1]) for i in range(0, len(fields), 2)}
    assert got["pairs"] == 523084815  # every (amax, x >= 0) pair of the domain
    assert got["one_step"] == 0
    assert got["negative"] == 0
    assert got["no_step"] > 0  # the refinement step is needed
