"""bench.py's reference arm on the host: the JSON line it prints carries the
keys of the benchmark contract, and under torchrun only rank 0 prints.  The
oracle's arithmetic is stubbed out here (identity), so the test checks the
line's shape, not a timing."""

import json

import pytest


@pytest.fixture
def fast_oracle(monkeypatch):
    from oracle import ns_oracle as O

    monkeypatch.setattr(O, "msign_ns", lambda x, **kw: x)


def test_reference_arm_line(monkeypatch, capsys, fast_oracle):
    import bench

    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3"])
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["steps"] == 3 and d["warmup"] == 3 and d["higher_is_better"] is False
    assert d["value"] == d["ms_per_step"] == d["cpu_baseline"]["value"] == d["e2e"]["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["rows"] == d["config"]["cols"] == 4096


def test_reference_arm_other_ranks_print_nothing(monkeypatch, capsys, fast_oracle):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3"])
    assert capsys.readouterr().out.strip() == ""


def test_warmup_below_three_is_refused():
    import bench

    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])
