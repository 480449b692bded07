"""The fused producers' selectable launch shapes: the whole producer parity
file (tests/test_gpu_producers.py: bit-exact codes, scales and row sums
against the oracle at every row width) run again in a process of its own
under each non-default shape of QOQ_FORCE_CONFIG, which is read once per
process: RMSNorm rows formed twice (prs=2) with the wider SiLU-gated CTA rows
(pst=2), and RMSNorm rows staged in shared memory (prs=3)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("cfg", ["prs=2,pst=2", "prs=3"])
def test_producer_parity_under_forced_shape(cfg):
    env = dict(os.environ, QOQ_FORCE_CONFIG=cfg)
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(HERE, "test_gpu_producers.py"), "-m", "gpu",
                        "-x", "-q", "-p", "no:cacheprovider"], cwd=os.path.dirname(HERE), env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and " passed" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
