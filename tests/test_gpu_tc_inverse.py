"""The tensor-core inverse build option (-DKDA_TC_INVERSE, libkda_tcinv.so).

Its split-role prefill computes T = (I + L)^-1 of each chunk with three rounds of tcgen05 MMAs,
T = (I + N^2)(I - N) D^-1 with N = D^-1 L_off, instead of the warp-level tf32 block merges. The
default build keeps the merges (they are faster: the MMA rounds add about 2,000 cycles to every
producer item). The option's library must still match the oracle on every kernel family."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tcinv_lib():
    from gated_delta_rule_62_b200 import build
    return build.build(tc_inverse=True)


def test_tc_inverse_build_matches_oracle_on_every_kernel_family(tcinv_lib):
    env = dict(os.environ, KDA_LIB=tcinv_lib)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_build_check.py"), "clean"],
                       capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "clean ok" in r.stdout
