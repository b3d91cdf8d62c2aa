"""bench.py's reference arm (the oracle timed on the host cores) on CPU: rank 0
prints one JSON line with the contract's keys, any other rank does no work."""
import json
import types

import bench


def _args(**kw):
    a = dict(workload="tiny_fp32", steps=2, warmup=1, cpu_budget=1.0)
    a.update(kw)
    return types.SimpleNamespace(**a)


def test_other_ranks_do_nothing(capsys):
    assert bench.run_reference(_args(), rank=1, world=2, local=1) is None
    assert capsys.readouterr().out == ""


def test_rank_zero_prints_one_reference_line(capsys):
    bench.run_reference(_args(), rank=0, world=1, local=0)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
