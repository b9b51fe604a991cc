"""Host-side parts of bench.py that need no GPU: the algorithmic-bytes
formula the bench reports against, the committed traffic record's source
check, the oracle baseline's fields and the clock-sample summary."""
import json
import os

import bench
from aq_inputs import LayerSpec
from conftest import ROOT


def test_algorithmic_bytes_of_the_default_layer():
    # codes 4096*512*2 + codebook 65536*16 + scales 2*4096 + x 2*4096 + y 2*4096
    assert bench.alg_bytes(LayerSpec(4096, 4096, 1, 16), 1) == 4194304 + 1048576 + 8192 + 8192 + 8192
    # batch grows x and y only
    assert (bench.alg_bytes(LayerSpec(4096, 4096, 1, 16), 16) - bench.alg_bytes(LayerSpec(4096, 4096, 1, 16), 1)
            == 15 * (2 * 4096 + 2 * 4096))
    # 2x8: two 8-bit codes per group, two 256-entry codebooks
    # (codes 11008*512*2, codebooks 2*256*16, scales and y 2*11008 each, x 2*4096)
    assert bench.alg_bytes(LayerSpec(11008, 4096, 2, 8), 1) == 11008 * 512 * 2 + 2 * 256 * 16 + 4 * 11008 + 2 * 4096


def test_traffic_record_only_while_the_sources_match(tmp_path, monkeypatch):
    import hashlib
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic_gemv_llama2-7b-1x16.json")))
    assert set(rec["per_launch_bytes"]) == {"1", "4", "16"} and rec["layer"] == "4096x4096"
    # a copy of the repository whose record was taken on its current sources
    fake = tmp_path / "repo"
    (fake / "profiles").mkdir(parents=True)
    h = hashlib.sha256()
    for f in rec["sources"]:
        dst = fake / f
        dst.parent.mkdir(parents=True, exist_ok=True)
        data = open(os.path.join(ROOT, f), "rb").read()
        dst.write_bytes(data)
        h.update(data)
    rec = dict(rec, sources_sha256=h.hexdigest())
    (fake / "profiles" / "traffic_gemv_llama2-7b-1x16.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(fake))
    for b in (1, 4, 16):
        assert bench.recorded_traffic("4096x4096", b) == rec["per_launch_bytes"][str(b)]
    assert bench.recorded_traffic("8192x8192", 1) is None  # another layer
    # once a kernel source changes, the record no longer counts
    gemv = next(f for f in rec["sources"] if f.endswith("gemv.cu"))
    (fake / gemv).write_bytes(open(os.path.join(ROOT, gemv), "rb").read() + b"\n// changed\n")
    assert bench.recorded_traffic("4096x4096", 1) is None


def test_cpu_baseline_fields():
    r = bench.cpu_baseline(bench.workload_units(bench.WORKLOAD), budget_s=0.05, single_budget_s=0.02)
    for k in ("value", "unit", "cores", "kind", "sample", "single_thread", "nproc", "cpu_model"):
        assert k in r
    assert r["kind"] == "oracle" and r["unit"] == "GB/s"
    assert r["value"] > 0 and r["single_thread"]["value"] > 0
    assert 1 <= r["cores"] <= r["nproc"]


def test_clock_summary_flags_throttle_reasons():
    s = bench.ClockSampler(0)
    s.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1900, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    out = s.summary()
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples"] == 3


def test_clock_summary_without_samples():
    s = bench.ClockSampler(0)
    s.lines = []
    out = s.summary()
    assert out["sm_mhz"] is None and out["samples"] == 0


def test_stored_bits_per_weight():
    # closed form 2.0 for 1x16 and 2x8; with codebooks and scales counted
    # the 1 MiB 1x16 codebook weighs on small layers
    for (o, i, K, B), stored in [((4096, 4096, 1, 16), 2.504), ((28672, 8192, 1, 16), 2.038),
                                 ((1024, 8192, 1, 16), 3.002), ((11008, 4096, 2, 8), 2.005)]:
        b = bench.bits_per_weight(LayerSpec(o, i, K, B))
        assert b["codes"] == 2.0 and b["stored"] == stored, (o, i, K, B, b)
    assert bench.bits_per_weight(LayerSpec(11008, 4096, 2, 16))["codes"] == 4.0
