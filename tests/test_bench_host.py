"""bench.py's host logic on CPU: the short runs that the default line carries
name real workloads, record a failing workload's error instead of stopping,
and keep each workload's own numbers; a per-launch traffic record counts
only for the kernel source it was captured on."""
import argparse
import hashlib
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _args():
    return argparse.Namespace(gpus=1, steps=2000, warmup=20, impl="own",
                              workload=bench.DEFAULT_WORKLOAD, layers=8, e2e_steps=1000,
                              cpu_budget=15.0, ref_budget=90.0, no_cpu=False, no_also=False)


def test_also_workloads_exist_and_exclude_the_default():
    names = [wl for wl, _, _ in bench.ALSO]
    assert len(names) == len(set(names))
    assert bench.DEFAULT_WORKLOAD not in names
    for wl, steps, nl in bench.ALSO:
        assert wl in bench.WORKLOADS
        assert steps >= 1 and nl >= 2  # at least two layers rotate (inputs larger than L2)


def test_run_also_records_errors_and_numbers(monkeypatch):
    seen = []

    def fake_run_own(a, wl, emit=True, extra=None):
        assert emit is False and a.no_cpu and a.warmup >= 3
        seen.append((wl, a.steps, a.layers))
        if wl == "decode-t1":
            raise RuntimeError("device lost")
        return {"value": 1.0, "ms_per_step": 2.0, "clocks": {"sm_mhz": 1965.0},
                "roofline": {"launch_ms": 0.5, "frac": 0.25, "unit": "GB/s", "peak": 6650.0}}

    monkeypatch.setattr(bench, "run_own", fake_run_own)
    args = _args()
    out = bench.run_also(args)
    assert [s[0] for s in seen] == [wl for wl, _, _ in bench.ALSO]
    assert [(s[1], s[2]) for s in seen] == [(st, nl) for _, st, nl in bench.ALSO]
    assert "device lost" in out["decode-t1"]["error"]
    ok = [wl for wl, _, _ in bench.ALSO if wl != "decode-t1"]
    for wl in ok:
        assert out[wl]["value"] == 1.0 and out[wl]["roofline_frac"] == 0.25
    # the caller's arguments are not modified
    assert args.steps == 2000 and args.layers == 8 and args.no_cpu is False


def test_traffic_records_apply_only_to_their_sources():
    """A record counts only for the kernel source it was captured on: the
    bench reports its bytes while the source's sha256 matches, else null."""
    found = 0
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        if not (name.startswith("traffic_") and name.endswith(".json")):
            continue
        found += 1
        d = json.load(open(os.path.join(ROOT, "profiles", name)))
        src = os.path.join(ROOT, d["source"])
        same = hashlib.sha256(open(src, "rb").read()).hexdigest() == d["source_sha256"]
        assert d["dram_bytes_per_launch"] > 0
        wl = name[len("traffic_"):-len(".json")]
        assert wl in bench.WORKLOADS
        got = bench.traffic_from_profile(wl)
        assert got == (d["dram_bytes_per_launch"] if same else None)
    assert found >= 1


def test_default_line_prints_once_with_the_short_runs(monkeypatch, capsys):
    calls = []

    def fake_run_own(a, wl, emit=True, extra=None):
        calls.append((wl, emit))
        if wl == "prefill-t8192":
            raise RuntimeError("out of memory")
        line = {"metric": "MoE-layer tokens/s", "value": 3.0, "ms_per_step": 1.0,
                "clocks": {"sm_mhz": 1965.0},
                "roofline": {"launch_ms": 0.5, "frac": 0.25, "unit": "GB/s", "peak": 6650.0}}
        if emit:
            print(json.dumps(line))
        return line

    monkeypatch.setattr(bench, "run_own", fake_run_own)
    monkeypatch.setattr("sys.argv", ["bench.py"])
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    bench.main()
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["value"] == 3.0
    assert calls[0] == (bench.DEFAULT_WORKLOAD, False)  # the headline runs first
    assert "out of memory" in d["other_workloads"]["prefill-t8192"]["error"]
    assert d["other_workloads"]["decode-t1"]["value"] == 3.0
    # --no-also: the headline alone
    calls.clear()
    monkeypatch.setattr("sys.argv", ["bench.py", "--no-also"])
    bench.main()
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1 and "other_workloads" not in json.loads(lines[0])
    assert calls == [(bench.DEFAULT_WORKLOAD, True)]
