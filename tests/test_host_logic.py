"""Host-side logic that the reported numbers depend on (CPU only, no GPU):
the binding's constants against include/ssd.h, the bench's algorithmic byte
model against hand counts, the traffic table lookup, and the roofline
arithmetic."""
import importlib.util
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_binding_constants_match_the_header():
    import mamba_ssd_scan_b200 as m
    text = open(os.path.join(ROOT, "include", "ssd.h")).read()
    defines = dict(re.findall(r"^#define (SSD_(?:FLAG|TC|DEBUG)_\w+) (\d+)", text, flags=re.M))
    assert defines, "no flags found in the header"
    for name, value in defines.items():
        assert getattr(m, name) == int(value), name
    # and every flag constant of the binding is declared in the header
    for name in dir(m):
        if re.match(r"SSD_(FLAG|TC|DEBUG)_", name):
            assert name in defines, name


@pytest.mark.parametrize("name,path_mb", [
    ("fwd_bf16_b4_L1024", 26.411008),
    ("fwd_bf16_b8_L4096_init", 304.08704),
    ("fwd_bf16_b1_L65536_G8", 1621.098496),
])
def test_path_bytes_are_the_inputs_and_y_once(name, path_mb):
    """The path's algorithmic bytes: x and y (b L H P bf16 each), B and C
    (b L G N bf16 each), dt (b L H bf16), the initial and final states (fp32)
    where the workload has them; no intermediate."""
    from mamba_ssd_scan_b200 import synthetic
    b = _bench()
    cfg = synthetic.FWD_CONFIGS[name]
    tok = cfg.batch * cfg.seqlen
    hand = (2 * tok * cfg.nheads * cfg.headdim * 2 + 2 * tok * cfg.ngroups * cfg.dstate * 2 +
            tok * cfg.nheads * 2)
    st = cfg.batch * cfg.nheads * cfg.headdim * cfg.dstate * 4
    hand += (st if cfg.init_state else 0) + (st if cfg.return_final else 0)
    got = b.algorithmic_cost(cfg, 2)["path"][0]
    assert got == hand
    assert abs(got / 1e6 - path_mb) < 1e-6


def test_kernel_bytes_count_the_fp32_and_hi_lo_states():
    """At L65536 G8: chunk_state writes the fp32 local states, state passing
    reads them and writes the hi / lo pair, chunk_scan reads the pair; 4 bytes
    per state element each way."""
    from mamba_ssd_scan_b200 import synthetic
    b = _bench()
    cfg = synthetic.FWD_CONFIGS["fwd_bf16_b1_L65536_G8"]
    cost = b.algorithmic_cost(cfg, 2)
    nc = cfg.seqlen // cfg.chunk
    states = cfg.batch * nc * cfg.nheads * cfg.headdim * cfg.dstate * 4
    x = cfg.batch * cfg.seqlen * cfg.nheads * cfg.headdim * 2
    bc = cfg.batch * cfg.seqlen * cfg.ngroups * cfg.dstate * 2
    vec = cfg.batch * cfg.nheads * nc * cfg.chunk * 4
    assert cost["state_passing"][0] == 2 * states + cfg.batch * cfg.nheads * nc * 4
    assert cost["chunk_state"][0] == x + bc + 2 * vec + states
    assert cost["chunk_scan"][0] == 2 * x + 2 * bc + 2 * vec + states


def test_traffic_lookup_follows_the_source_digest(tmp_path, monkeypatch):
    b = _bench()
    # an entry with a digest that no source hashes to is never reported
    assert b.measured_traffic("chunk_scan", "no_such_workload") is None
    assert b.measured_traffic("no_such_kernel", "fwd_bf16_b1_L65536_G8") is None
    # a table whose digest matches the kernel's sources is read back as read + write
    import hashlib
    h = hashlib.sha256()
    for f in b.KERNEL_SOURCES["state_passing"]:
        with open(os.path.join(ROOT, "mamba_ssd_scan_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    digest = h.hexdigest()[:16]
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "dram_traffic.md").write_text(
        "| workload | kernel | source | read | write | ns |\n|---|---|---|---|---|---|\n"
        f"| wl | state_passing | {digest} | 100 | 23 | 5 |\n"
        "| wl | state_passing | 0000000000000000 | 7 | 7 | 5 |\n")
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    # the sources are still read from the package, the table from the temporary root
    real = os.path.join(ROOT, "mamba_ssd_scan_b200")
    os.symlink(real, tmp_path / "mamba_ssd_scan_b200")
    assert b.measured_traffic("state_passing", "wl") == 123


def test_roofline_names_the_bound_and_its_fraction():
    b = _bench()
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "source": "measured"}
    # 6 GB in 1 ms at 6 TB/s: exactly the copy bandwidth, memory-bound
    r = b.roofline_entry("k", (6e9, 1e12), 1.0, peaks, {"sm_mhz": 1965.0}, True, "wl")
    assert r["bound"] == "hbm" and abs(r["frac"] - 1.0) < 1e-12 and r["unit"] == "GB/s"
    # 1.5e12 FLOP in 2 ms on the tensor cores: half the peak, compute-bound
    r = b.roofline_entry("k", (1e6, 1.5e12), 2.0, peaks, {"sm_mhz": 1965.0}, True, "wl")
    assert r["bound"] == "tensor" and abs(r["frac"] - 0.5) < 1e-12 and r["unit"] == "TFLOP/s"
