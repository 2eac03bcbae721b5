"""Failure detection without a GPU fault: a kernel whose bounded wait runs out
returns an error status the host reads, and the context stays usable.

The library's test hook (ssd_debug_set_withhold, read by the host launcher)
makes one producer withhold one hand-off:
  - the convolution's producer warp its first tile: the consumers' waits on
    that tile's mbarrier give up after their iteration limit;
  - the forward's tensor-core chunk_scan the decays of the first head of its
    second chunk: that CTA's workers give up their wait and the CTA stops;
  - the single-pass forward (SSD_FLAG_SINGLE_PASS) the state leaving its first
    run of tiles (512 tokens): the CTA of the second run that waits for it
    polls the carry ring until its limit (about a second), raises the abort
    word, and every CTA stops.
The status call must then report SSD_ERR_TIMEOUT, and the same process runs
the operation again with the hook off and checks it against the oracle.  Each
case runs in a child process with a time limit."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PRELUDE = r"""
import os, sys, torch
sys.path.insert(0, ROOT); sys.path.insert(0, os.path.join(ROOT, "tests"))
import mamba_ssd_scan_b200 as ssd
from mamba_ssd_scan_b200 import synthetic
import oracle
from tolerance import assert_close
"""

CONV = r"""
inp = synthetic.make_conv_inputs(1, 64, 64, 4, torch.float32, seed=2)
d = {k: v.cuda() for k, v in inp.items()}
assert ssd.ssd_conv1d_check_status() == 0
ssd.ssd_debug_set_withhold(ssd.SSD_DEBUG_CONV_TILE, 0)
ssd.ssd_causal_conv1d(d["x"], d["weight"], d["bias"], d["init_state"])
st = ssd.ssd_conv1d_check_status()
assert st == 4, f"expected SSD_ERR_TIMEOUT (4), got {st}"
ssd.ssd_debug_set_withhold(ssd.SSD_DEBUG_CONV_TILE, -1)
y = ssd.ssd_causal_conv1d(d["x"], d["weight"], d["bias"], d["init_state"])
assert ssd.ssd_conv1d_check_status() == 0
yo, _ = oracle.load().causal_conv1d(inp["x"], inp["weight"], inp["bias"], inp["init_state"], True)
assert_close(y, yo, torch.float32, "after the timeout")
print("TIMEOUT-OK")
"""

# bf16, four chunks per sequence, two sequences.  MODE: "workspace" or
# "no_alloc" (the scratch inside the library) for the default three-kernel
# path; "single_pass" for the one-kernel forward.
FWD = r"""
b, L, H, P, N, G, Q = 2, 1024, 4, 64, 64, 1, 256
inp = synthetic.make_fwd_inputs(b, L, H, P, N, G, torch.bfloat16, seed=11, init_state=True)
d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
NO_ALLOC = MODE == "no_alloc"
FLAGS = ssd.SSD_FLAG_SINGLE_PASS if MODE == "single_pass" else 0
HOOK = ssd.SSD_DEBUG_FWD_CARRY if MODE == "single_pass" else ssd.SSD_DEBUG_SCAN_DECAYS
steps = ssd.tensor_core_steps(b, L, H, P, N, G, Q, torch.bfloat16, flags=FLAGS)
assert ("fused" in steps) == (MODE == "single_pass") and "chunk_scan" in steps, steps

def run():
    if NO_ALLOC:
        y = torch.empty_like(d["x"])
        ssd.ssd_fwd_no_alloc(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"], Q,
                             d["init_state"], y=y, flags=FLAGS)
        return y, ssd.ssd_fwd_no_alloc_check_status(d["x"], d["B"], Q, flags=FLAGS)
    ws = torch.empty(ssd.ssd_fwd_workspace_size(b, L, H, P, N, G, Q, torch.bfloat16, flags=FLAGS),
                     dtype=torch.uint8, device="cuda")
    y = ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"], Q,
                    d["init_state"], workspace=ws, flags=FLAGS)
    return y, ssd.ssd_fwd_check_status(d["x"], d["B"], Q, ws, flags=FLAGS)

y, st = run()
assert st == 0, f"clean run: status {st}"
ssd.ssd_debug_set_withhold(HOOK, 0 if MODE == "single_pass" else 1)
y, st = run()
assert st == 4, f"expected SSD_ERR_TIMEOUT (4), got {st}"
ssd.ssd_debug_set_withhold(HOOK, -1)
y, st = run()
assert st == 0, f"after the timeout: status {st}"
yo, _ = oracle.load().ssd_fwd(**inp)
assert_close(y, yo, torch.bfloat16, "y after the timeout")
print("TIMEOUT-OK")
"""


def _child(body, mode=""):
    code = "ROOT = %r\nMODE = %r\n" % (ROOT, mode) + PRELUDE + body
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=240)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "TIMEOUT-OK" in r.stdout


def test_withheld_tile_times_out_and_context_survives():
    _child(CONV)


def test_withheld_decays_time_out_and_context_survives():
    _child(FWD, "workspace")


def test_no_alloc_reports_the_timeout():
    _child(FWD, "no_alloc")


def test_single_pass_withheld_carry_times_out_and_context_survives():
    _child(FWD, "single_pass")
