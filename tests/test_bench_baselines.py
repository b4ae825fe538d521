"""The bench's oracle baselines run on the host alone (CPU only): the plain step's and the
gated layer's, on a small configuration, with a bounded sample and the contract's keys.
The plain step's leg also checks the last timed step's lists and outputs; here it is fed
the oracle's own results (everything equal, errors zero) and then one planted wrong list."""
import numpy as np
import torch

import bench
import oracle as O
import synth


def _check(r):
    assert {"value", "unit", "cores", "kind", "sample"} <= set(r)
    assert r["kind"] == "oracle" and r["unit"] == bench.UNIT and r["value"] > 0 and r["cores"] >= 1


def _oracle_as_gpu(cfg, host, heads):
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    idx = np.full((len(heads), T, T), -1, np.int32)
    cnt = np.zeros((len(heads), T), np.int32)
    outs = {n: np.zeros((len(heads), lay.n_pad, cfg.D)) for n in ("out", "dq", "dk", "dv")}
    for hi, h in enumerate(heads):
        t = {n: O.tile(host[n][0, h].double().numpy(), lay) for n in ("q", "k", "v", "do")}
        tr = O.route_head(t["q"], t["k"], lay.valid, cfg.top_k, cfg.top_p)
        for i, l in enumerate(tr.lists):
            idx[hi, i, :len(l)] = l
            cnt[hi, i] = len(l)
        outs["out"][hi] = O.attention_forward_head(t["q"], t["k"], t["v"], tr.lists, lay.valid)[0]
        outs["dq"][hi], outs["dk"][hi], outs["dv"][hi] = O.attention_backward_head(
            t["q"], t["k"], t["v"], t["do"], tr.lists, lay.valid)
    g = {"heads": heads, "idx": torch.from_numpy(idx), "cnt": torch.from_numpy(cnt)}
    g.update({n: torch.from_numpy(v) for n, v in outs.items()})
    return g, int(cnt.sum())


def test_cpu_baselines_small():
    cfg = synth.small_config("tiny_b", 1, 4, 64, (8, 16, 16), 4, 0.9)
    host = synth.make_inputs(cfg, 0)
    heads = bench.oracle_heads(cfg.H)
    assert heads == [0, 1, 2, 3]
    gpu, ntiles = _oracle_as_gpu(cfg, host, heads)
    base, par = bench.cpu_baseline(cfg, host, gpu, ntiles, seconds=0.5)
    _check(base)
    assert base["extrapolated"] and base["host_cpus"] >= 1
    assert par["mismatch_rows"] == 0 and par["tie_rows"] == 0 and par["equal_rows"] == par["rows"] == 4 * 32
    assert all(v < 1e-12 for v in par["max_abs"].values()) and {"out", "dq"} <= set(par["max_abs"])
    # a planted wrong list (one block swapped for an unselected one) is a mismatch, not a tie
    row = gpu["idx"][1, 5, :gpu["cnt"][1, 5]].numpy()
    spare = next(j for j in range(32) if j not in set(row.tolist()))
    gpu["idx"][1, 5, 0] = spare
    gpu["idx"][1, 5, :gpu["cnt"][1, 5]] = torch.from_numpy(np.sort(gpu["idx"][1, 5, :gpu["cnt"][1, 5]].numpy()))
    _, par = bench.cpu_baseline(cfg, host, gpu, ntiles, seconds=0.5)
    assert par["mismatch_rows"] == 1 and par["equal_rows"] == 4 * 32 - 1
    r = bench.cpu_baseline_gated(cfg, host, synth.make_gate(cfg), seconds=0.5)
    _check(r)
    assert "coarse branch" in r["sample"]


def test_valid_counts_per_cube():
    # 5 x 6 x 7 latent: cubes along t hold 4 and 1 rows, along h 4 and 2, along w 4 and 3
    v = bench.cube_valid_counts((5, 6, 7))
    assert len(v) == 2 * 2 * 2 and v[0] == 64 and v[-1] == 1 * 2 * 3 and sum(v) == 5 * 6 * 7
