"""Failure detection without a GPU fault: a kernel whose bounded wait runs out
returns an error status the host reads, and the context stays usable.

The convolution's producer warp is told (SSD_DEBUG_WITHHOLD_TILE, read by
the host launcher) to withhold its first tile: the consumers' waits on that
tile's mbarrier give up after their iteration limit (about a second), every
role stops, the copies in flight land, and ssd_conv1d_check_status reports
SSD_ERR_TIMEOUT.  The same process then runs the convolution normally and
checks it against the oracle.  Runs in a child process with a time limit."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import os, sys, torch
sys.path.insert(0, ROOT); sys.path.insert(0, os.path.join(ROOT, "tests"))
import mamba_ssd_scan_b200 as ssd
from mamba_ssd_scan_b200 import synthetic
import oracle
from tolerance import assert_close
inp = synthetic.make_conv_inputs(1, 64, 64, 4, torch.float32, seed=2)
d = {k: v.cuda() for k, v in inp.items()}
assert ssd.ssd_conv1d_check_status() == 0
os.environ["SSD_DEBUG_WITHHOLD_TILE"] = "0"
ssd.ssd_causal_conv1d(d["x"], d["weight"], d["bias"], d["init_state"])
st = ssd.ssd_conv1d_check_status()
assert st == 4, f"expected SSD_ERR_TIMEOUT (4), got {st}"
del os.environ["SSD_DEBUG_WITHHOLD_TILE"]
y = ssd.ssd_causal_conv1d(d["x"], d["weight"], d["bias"], d["init_state"])
assert ssd.ssd_conv1d_check_status() == 0
yo, _ = oracle.load().causal_conv1d(inp["x"], inp["weight"], inp["bias"], inp["init_state"], True)
assert_close(y, yo, torch.float32, "after the timeout")
print("TIMEOUT-OK")
"""


def test_withheld_tile_times_out_and_context_survives():
    code = "ROOT = %r\n" % ROOT + CHILD
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=180)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "TIMEOUT-OK" in r.stdout
