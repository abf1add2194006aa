"""The kernels selected by environment switches, read once per process: the
TMEM-resident tcgen05 state chains (SF_GDN_CHAIN=tcgen05), the warp-level
gradient kernel (SF_GDN_GRAD=warp) and the warp-level Out kernel
(SF_GDN_OUT=warp).  Each runs in a child process through the
same parity, bit-identity and live-state tests as the default kernels."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SELECT = ("bf16_small or chunk_sizes or config2 or bit_identical_to_standalone or "
          "bounded_memory_chain_bit_identical or live_state_standalone")


@pytest.mark.parametrize("env", [{"SF_GDN_CHAIN": "tcgen05"}, {"SF_GDN_GRAD": "warp"}, {"SF_GDN_OUT": "warp"}],
                         ids=["tcgen05_chains", "warp_grad", "warp_out"])
def test_switched_kernels(env):
    e = dict(os.environ)
    e.update(env)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_parity.py", "tests/test_gpu_pipeline.py", "tests/test_gpu_live_state.py",
           "-k", SELECT]
    r = subprocess.run(cmd, cwd=ROOT, env=e, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout, r.stdout[-2000:]
