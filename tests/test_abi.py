"""The C-ABI library loads, exports every function include/ssd.h declares, and
rejects bad arguments before touching the GPU (CPU only: no compute calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


@pytest.fixture(scope="module")
def lib():
    from mamba_ssd_scan_b200 import build
    build.build()
    import mamba_ssd_scan_b200 as m
    return m.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(ssd_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ("ssd_fwd", "ssd_fwd_workspace_size", "ssd_state_update",
                     "ssd_status_string", "ssd_chunk_cumsum", "ssd_chunk_state",
                     "ssd_state_passing", "ssd_chunk_scan", "ssd_fwd_check_status",
                     "ssd_state_passing_hilo", "ssd_chunk_scan_hilo"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(os.path.join(ROOT, "mamba_ssd_scan_b200", "libssd_b200.so"))
    missing = [n for n in declared_functions() if not hasattr(raw, n)]
    assert not missing, f"declared but not exported: {missing}"


def test_tensor_core_dispatch_query(lib):
    import torch

    import mamba_ssd_scan_b200 as m
    # bf16: chunk_state and chunk_scan on the tensor cores (fp32 chunk states,
    # entering chunk_scan as hi / lo bf16 halves)
    assert m.tensor_core_steps(4, 1024, 24, 64, 64, 1, 256) == {"chunk_state", "chunk_scan"}
    assert m.tensor_core_steps(1, 65536, 80, 64, 128, 8, 256) == {"chunk_state", "chunk_scan"}
    assert m.tensor_core_steps(1, 300, 4, 64, 128, 2, 128) == {"chunk_state", "chunk_scan"}
    # one head per group: chunk_state's tile takes 128 / headdim heads of a group
    assert m.tensor_core_steps(1, 300, 4, 64, 128, 4, 128) == {"chunk_scan"}
    assert m.tensor_core_steps(4, 1024, 24, 64, 64, 1, 256, torch.float32) == set()
    assert m.tensor_core_steps(4, 1024, 24, 64, 64, 1, 256, flags=m.SSD_FLAG_CUDA_CORES) == set()
    assert m.tensor_core_steps(4, 1024, 24, 64, 64, 1, 256, flags=m.SSD_FLAG_SPLIT_STEPS) == {
        "chunk_state", "chunk_scan"}
    # the opt-in bf16-states mode also takes the tensor-core chunk_scan
    assert m.tensor_core_steps(4, 1024, 24, 64, 64, 1, 256, flags=m.SSD_FLAG_BF16_STATES) == {
        "chunk_state", "chunk_scan"}
    # chunk_scan's tensor-core kernel takes headdim 64 and dstate 64 / 128 only
    assert m.tensor_core_steps(1, 512, 2, 128, 256, 1, 256) == {"chunk_state"}
    # chunk 64: neither tensor-core step kernel
    assert m.tensor_core_steps(1, 512, 4, 64, 128, 4, 64) == set()
    # the single-pass kernel (opt-in) tiles the sequence its own way: any chunk
    sp = m.SSD_FLAG_SINGLE_PASS
    assert m.tensor_core_steps(1, 512, 4, 64, 128, 4, 64, flags=sp) == {
        "chunk_state", "chunk_scan", "fused"}
    assert m.tensor_core_steps(4, 1024, 24, 64, 64, 1, 256, flags=sp) == {
        "chunk_state", "chunk_scan", "fused"}
    assert m.tensor_core_steps(1, 512, 4, 64, 128, 4, 64, flags=sp | m.SSD_FLAG_SPLIT_STEPS) == set()
    assert m.tensor_core_steps(1, 512, 2, 128, 256, 1, 256, flags=sp) == {"chunk_state"}


def test_status_strings(lib):
    import mamba_ssd_scan_b200 as m
    assert m.ssd_status_string(0) == "SSD_OK"
    assert m.ssd_status_string(2) == "SSD_ERR_UNSUPPORTED"
    assert "sm_100a" in m.ssd_version()


def _args(**kw):
    import mamba_ssd_scan_b200 as m
    a = m.SsdFwdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk = 1, 512, 4, 64, 64, 1, 256
    a.dtype = m.SSD_BF16
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_workspace_size_is_host_only(lib):
    import mamba_ssd_scan_b200 as m
    # default (three kernels): header + dt + cumA (1*4*2*256 fp32 each) + fp32
    # chunk states 1*2*4*64*64 + their hi / lo bf16 halves
    assert lib.ssd_fwd_workspace_size(ctypes.byref(_args())) == 256 + 8192 + 8192 + 131072 + 131072
    a = _args(flags=m.SSD_FLAG_SPLIT_STEPS)
    assert lib.ssd_fwd_workspace_size(ctypes.byref(a)) == 256 + 8192 + 8192 + 131072 + 131072
    # the CUDA cores form the state term from the fp32 states: no halves
    a = _args(flags=m.SSD_FLAG_SPLIT_STEPS | m.SSD_FLAG_CUDA_CORES)
    assert lib.ssd_fwd_workspace_size(ctypes.byref(a)) == 256 + 8192 + 8192 + 131072
    # bf16-states mode: the chunk states in bf16, no halves
    a = _args(flags=m.SSD_FLAG_BF16_STATES)
    assert lib.ssd_fwd_workspace_size(ctypes.byref(a)) == 256 + 8192 + 8192 + 65536
    # single pass: header (256 B), the ring's reader counts (2*1*4 ints, in
    # 256 B) and a two-slot ring of 1*4 states of 64*64 fp32
    a = _args(flags=m.SSD_FLAG_SINGLE_PASS)
    assert lib.ssd_fwd_workspace_size(ctypes.byref(a)) == 256 + 256 + 2 * 4 * 64 * 64 * 4
    assert lib.ssd_fwd_workspace_size(None) == 0
    assert lib.ssd_fwd_workspace_size(ctypes.byref(_args(nheads=3, ngroups=2))) == 0


@pytest.mark.parametrize("bad,status", [
    (dict(batch=0), 1), (dict(seqlen=-1), 1), (dict(nheads=6, ngroups=4), 1),
    (dict(dtype=7), 1), (dict(chunk=512), 2), (dict(dstate=66), 2), (dict(dstate=512), 2),
    (dict(headdim=6), 2),
])
def test_fwd_rejects_bad_sizes(lib, bad, status):
    assert lib.ssd_fwd(ctypes.byref(_args(**bad)), None) == status


def test_fwd_rejects_null_and_host_pointers(lib):
    # null required pointers
    assert lib.ssd_fwd(ctypes.byref(_args()), None) == 1
    # host memory is never accepted as device memory
    buf = ctypes.create_string_buffer(1 << 16)
    p = ctypes.addressof(buf)
    a = _args(x=p, dt=p, A=p, B=p, C=p, y=p, workspace=p, workspace_bytes=1 << 16)
    assert lib.ssd_fwd(ctypes.byref(a), None) == 1
    assert lib.ssd_fwd(None, None) == 1


def test_state_update_rejects_bad_args(lib):
    import mamba_ssd_scan_b200 as m
    a = m.SsdStateUpdateArgs()
    a.batch, a.nheads, a.headdim, a.dstate, a.ngroups, a.dtype = 2, 4, 64, 128, 1, m.SSD_BF16
    assert lib.ssd_state_update(ctypes.byref(a), None) == 1  # null pointers
    a.dstate = 48
    assert lib.ssd_state_update(ctypes.byref(a), None) == 2
    a.dstate, a.ngroups = 128, 3
    assert lib.ssd_state_update(ctypes.byref(a), None) == 1


def test_conv1d_rejects_bad_args(lib):
    import mamba_ssd_scan_b200 as ssd
    a = ssd.SsdConv1dArgs()
    a.batch, a.seqlen, a.channels, a.width, a.dtype, a.activation = 2, 64, 16, 4, 1, 1
    assert lib.ssd_causal_conv1d(None, None) == 1
    assert lib.ssd_causal_conv1d(ctypes.byref(a), None) == 1        # null pointers
    a.width = 9
    assert lib.ssd_causal_conv1d(ctypes.byref(a), None) == 2        # width beyond 8
    a.width, a.channels = 4, 12
    assert lib.ssd_causal_conv1d(ctypes.byref(a), None) == 2        # bf16 channels % 8
    a.channels, a.seqlen = 16, 0
    assert lib.ssd_causal_conv1d(ctypes.byref(a), None) == 1        # empty sequence
    u = ssd.SsdConv1dUpdateArgs()
    u.batch, u.channels, u.width, u.dtype = 2, 16, 4, 0
    assert lib.ssd_conv1d_update(ctypes.byref(u), None) == 1        # null pointers
    u.width = 0
    assert lib.ssd_conv1d_update(ctypes.byref(u), None) == 1
    u.width, u.channels = 4, 6
    assert lib.ssd_conv1d_update(ctypes.byref(u), None) == 2        # fp32 channels % 4
    u.width = 9
    assert lib.ssd_conv1d_update(ctypes.byref(u), None) == 2        # width beyond 8


def test_bwd_rejects_bad_args(lib):
    import mamba_ssd_scan_b200 as ssd
    a = ssd.SsdBwdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk = 1, 256, 4, 64, 64, 1, 256
    a.dtype = 1
    assert lib.ssd_bwd(None, None) == 1
    assert lib.ssd_bwd_workspace_size(ctypes.byref(a)) > 0
    assert lib.ssd_bwd(ctypes.byref(a), None) == 1               # null pointers
    a.chunk = 100
    assert lib.ssd_bwd_workspace_size(ctypes.byref(a)) == 0
    assert lib.ssd_bwd(ctypes.byref(a), None) == 2               # chunk not a multiple of 64
    a.chunk, a.headdim = 256, 256
    assert lib.ssd_bwd(ctypes.byref(a), None) == 2               # headdim beyond 128
    a.headdim, a.dstate = 128, 128
    assert lib.ssd_bwd(ctypes.byref(a), None) == 2               # tiles beyond shared memory
    a.dstate, a.ngroups = 64, 3
    assert lib.ssd_bwd(ctypes.byref(a), None) == 1               # heads not divisible by groups


def test_selective_scan_rejects_bad_args(lib):
    import mamba_ssd_scan_b200 as ssd
    a = ssd.SsdSelectiveScanArgs()
    a.batch, a.seqlen, a.channels, a.dstate, a.chunk, a.dtype = 1, 64, 32, 16, 64, 0
    assert lib.ssd_selective_scan(None, None) == 1
    assert lib.ssd_selective_scan_workspace_size(ctypes.byref(a)) > 0
    assert lib.ssd_selective_scan(ctypes.byref(a), None) == 1     # null pointers
    a.dstate = 6
    assert lib.ssd_selective_scan(ctypes.byref(a), None) == 2     # dstate not a multiple of 4
    a.dstate = 36
    assert lib.ssd_selective_scan(ctypes.byref(a), None) == 2     # dstate beyond 32
    a.dstate, a.chunk = 32, 256
    assert lib.ssd_selective_scan_workspace_size(ctypes.byref(a)) == 0   # chunk * dstate > 4096
    u = ssd.SsdSelectiveStateUpdateArgs()
    u.batch, u.channels, u.dstate, u.dtype = 2, 32, 16, 1
    assert lib.ssd_selective_state_update(ctypes.byref(u), None) == 1   # null pointers
    u.dstate = 40
    assert lib.ssd_selective_state_update(ctypes.byref(u), None) == 2


def test_gated_rmsnorm_rejects_bad_args(lib):
    import mamba_ssd_scan_b200 as ssd
    a = ssd.SsdGatedRmsnormArgs()
    a.rows, a.channels, a.group, a.dtype, a.eps = 4, 64, 32, 1, 1e-5
    assert lib.ssd_gated_rmsnorm(None, None) == 1
    assert lib.ssd_gated_rmsnorm(ctypes.byref(a), None) == 1      # null pointers
    a.group = 48
    assert lib.ssd_gated_rmsnorm(ctypes.byref(a), None) == 2      # channels % group
    a.group = 4
    assert lib.ssd_gated_rmsnorm(ctypes.byref(a), None) == 2      # bf16 group % 8
    a.dtype = 0
    assert lib.ssd_gated_rmsnorm(ctypes.byref(a), None) == 1      # fp32 group 4 fine: null pointers
    a.group, a.eps = 32, -1.0
    assert lib.ssd_gated_rmsnorm(ctypes.byref(a), None) == 1      # negative eps
    a.eps, a.rows = 1e-5, 0
    assert lib.ssd_gated_rmsnorm(ctypes.byref(a), None) == 1      # no rows


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """With the shared library absent the binding raises on the first call;
    no entry point falls back to another implementation."""
    import torch
    import mamba_ssd_scan_b200 as ssd
    monkeypatch.setattr(ssd, "_lib", None)
    monkeypatch.setattr(ssd, "_LIB_FILE", str(tmp_path / "libssd_b200.so"))
    with pytest.raises(RuntimeError, match="missing"):
        ssd.load_library()
    x = torch.zeros((1, 8, 2, 16))
    with pytest.raises(RuntimeError, match="missing"):
        ssd.ssd_fwd(x, torch.zeros((1, 8, 2)), torch.zeros(2), torch.zeros((1, 8, 1, 16)),
                    torch.zeros((1, 8, 1, 16)), chunk=8)


def test_no_alloc_scratch_size_matches_the_header(lib):
    import mamba_ssd_scan_b200 as ssd
    text = open(os.path.join(ROOT, "include", "ssd.h")).read()
    m = re.search(r"#define SSD_NO_ALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", text)
    assert m, "SSD_NO_ALLOC_SCRATCH_BYTES not found in the header"
    assert ssd.ssd_fwd_no_alloc_scratch_bytes() == int(m.group(1)) << int(m.group(2))


def test_no_alloc_status_rejects_sizes_on_the_host(lib):
    # beyond the built-in buffer, and invalid sizes: answered before any
    # device access
    a = _args(batch=8, seqlen=4096, nheads=32, headdim=64, dstate=128)
    assert lib.ssd_fwd_no_alloc_check_status(ctypes.byref(a), None) == 2  # UNSUPPORTED
    assert lib.ssd_fwd_no_alloc_check_status(ctypes.byref(_args(batch=0)), None) == 1
    assert lib.ssd_fwd_no_alloc_check_status(None, None) == 1
    # ssd_fwd_no_alloc itself rejects the oversize call before launching
    assert lib.ssd_fwd_no_alloc(ctypes.byref(a), None) in (1, 2)
