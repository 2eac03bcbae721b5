"""ssd_fwd_no_alloc: the forward scan for callers that cannot allocate device
memory (plugins handed only their input/output buffers, latency-critical code
that must not risk a cudaMalloc's synchronisation).  Its scratch is a fixed
buffer inside the library, so its results must match ssd_fwd with a
caller-provided workspace, call after call, with the buffer reused.

This file sorts last so that a run stopping at the first failure has already
run every other test.
"""
import pytest
import torch

import mamba_ssd_scan_b200 as ssd
from mamba_ssd_scan_b200 import synthetic
from tolerance import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(shape, dtype, seed):
    b, L, H, P, N, G = shape
    inp = synthetic.make_fwd_inputs(b, L, H, P, N, G, dtype, seed=seed, init_state=True)
    return {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}


@pytest.mark.parametrize("shape,dtype,chunk", [
    ((4, 1024, 24, 64, 64, 1), torch.bfloat16, 256),   # the headline workload's shape
    ((1, 256, 4, 16, 16, 1), torch.float32, 64),       # the small fp32 workload's shape
])
def test_no_alloc_matches_ssd_fwd_twice(shape, dtype, chunk):
    b, L, H, P, N, G = shape
    for call, seed in enumerate((101, 202)):  # two calls in a row share the buffer
        d = _inputs(shape, dtype, seed)
        y_ref, f_ref = ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"],
                                   chunk, d["init_state"], return_final_state=True)
        y = torch.full_like(d["x"], float("nan"))
        fin = torch.full((b, H, P, N), float("nan"), device=DEV)
        ssd.ssd_fwd_no_alloc(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"],
                             chunk, d["init_state"], y=y, final_state=fin)
        torch.cuda.synchronize()
        assert_close(y, y_ref.double().cpu().numpy(), dtype, f"y, call {call}")
        assert_close(fin, f_ref.double().cpu().numpy(), dtype, f"final state, call {call}")


def test_no_alloc_rejects_sizes_beyond_the_buffer():
    # 8 x 4096 tokens, 32 heads of 64 x 128: ~84 MB of scratch, more than 16 MiB
    d = _inputs((8, 4096, 32, 64, 128, 1), torch.bfloat16, 7)
    y = torch.full_like(d["x"], 3.0)
    with pytest.raises(ssd.SsdError) as e:
        ssd.ssd_fwd_no_alloc(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"], 256,
                             d["init_state"], y=y)
    assert e.value.status == ssd.SSD_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (y == 3.0).all()  # nothing was launched
