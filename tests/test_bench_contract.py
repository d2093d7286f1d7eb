"""The benchmark's JSON line (CPU): the reference arm (the oracle, timed) prints one line with
the keys the contract names, on a tiny sample."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0", "--ref-tokens", "16"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["value"] == d["value"]


def _bench():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def test_per_pipe_bound_names_the_binding_pipe():
    """The derived ALU bound: each pipe's Gnormal/s is SMs x clock x (ops per clock) / (ops per
    normal), and the smallest names the binding pipe.  With 18 widening multiplies per block of
    four normals (two results each) the integer multiply binds the forward and the draw
    reduction; the LM head's long consumer makes issue bind."""
    b = _bench()
    bounds, binding, ops = b.alu_bounds("fwd", 148, 1965.0)
    assert binding == "imad" and ops["imad"] == 18 * 2 / 4
    assert abs(bounds["imad"] - 148 * 1965e6 * 64 / 9 / 1e9) < 0.1
    assert abs(bounds["xu"] - 148 * 1965e6 * 16 / 2 / 1e9) < 0.1
    assert b.alu_bounds("ghat", 148, 1965.0)[1] == "imad"
    hb, hbind, _ = b.alu_bounds("lmhead", 148, 1965.0)
    assert hbind == "issue" and hb["issue"] < hb["imad"]
    # a longer consumer never raises a bound; a faster clock raises every bound in proportion
    assert all(hb[p] <= bounds[p] for p in bounds)
    b2 = b.alu_bounds("fwd", 148, 2 * 1965.0)[0]
    assert all(abs(b2[p] - 2 * bounds[p]) < 0.2 for p in bounds)


def test_measured_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    """A DRAM figure from an ncu capture is tied to the digest of the sources that built the
    kernel: with the current digest it is reported, with any other it is not."""
    b = _bench()
    files = ("dust_fwd.cu", "dust_device.cuh", "dust_internal.h")
    digest = b.source_digest(files)
    monkeypatch.setattr(b, "MEASURED_TRAFFIC", {("k", "w"): (123, files, digest, "p.md")})
    assert b.measured_traffic("k", "w") == (123, "p.md")
    assert b.measured_traffic("k", "other") == (None, None)
    monkeypatch.setattr(b, "MEASURED_TRAFFIC", {("k", "w"): (123, files, "0" * 16, "p.md")})
    assert b.measured_traffic("k", "w") == (None, None)

