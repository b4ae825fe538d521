"""The bench's oracle baselines run on the host alone (CPU only): the plain step's and the
gated layer's, on a small configuration, with a bounded sample and the contract's keys."""
import bench
import synth


def _check(r):
    assert set(r) == {"value", "unit", "cores", "kind", "sample"}
    assert r["kind"] == "oracle" and r["unit"] == bench.UNIT and r["value"] > 0 and r["cores"] >= 1


def test_cpu_baselines_small():
    cfg = synth.small_config("tiny_b", 1, 1, 64, (8, 16, 16), 4, 0.9)
    host = synth.make_inputs(cfg, 0)
    _check(bench.cpu_baseline(cfg, host, seconds=0.5))
    r = bench.cpu_baseline_gated(cfg, host, synth.make_gate(cfg), seconds=0.5)
    _check(r)
    assert "coarse branch" in r["sample"]
