"""Host-side pieces of the bench, on CPU: the clock summary taken during the
timed region (median SM clock, throttle reasons) and the ncu traffic record,
which is reported only for the workload it was taken on and only while the
scorer's sources are the ones it was captured from."""
import json
import os
import shutil
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _sampler(rows):
    s = bench.ClockSampler.__new__(bench.ClockSampler)   # no nvidia-smi process
    s.samples = rows
    s.proc = None
    return s


def _row(sm, power, hw="Not Active", hw_thermal="Not Active", sw_thermal="Not Active", power_cap="Not Active"):
    return ["2026/01/01 00:00:00.000", "0", str(sm), "1965", str(power), "0x0", hw, hw_thermal, sw_thermal, power_cap]


def test_clock_summary_inside_the_window():
    rows = [(1.0, _row(1800, 500.5, power_cap="Active")),
            (1.1, _row(1900, 600.0)),
            (1.2, _row(1950, 610.0, hw_thermal="Active")),
            (5.0, _row(500, 100.0, hw="Active"))]          # after the timed region: ignored
    d = _sampler(rows).summary(0.9, 1.3)
    assert d["samples"] == 3
    assert d["sm_mhz"] == 1900.0 and d["sm_max_mhz"] == 1965.0
    assert d["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert d["power_w_max"] == 610.0


def test_clock_summary_unparsable_fields_and_no_samples():
    rows = [(1.0, _row("[N/A]", "[N/A]")), (1.1, _row(1700, 400.0))]
    d = _sampler(rows).summary(0.0, 2.0)
    assert d["sm_mhz"] == 1700.0 and d["power_w_max"] == 400.0 and d["reasons"] == []
    d = _sampler([]).summary(0.0, 1.0)
    assert d["samples"] == 0 and d["sm_mhz"] is None and d["reasons"] == ["nvidia-smi unavailable"]


def _tree(tmp_path):
    """A copy of the scorer sources and an empty profiles folder."""
    src = os.path.join(ROOT, "rope_aware_key_b200", "csrc")
    dst = tmp_path / "rope_aware_key_b200" / "csrc"
    shutil.copytree(src, dst)
    (tmp_path / "profiles").mkdir()
    return dst


def _record(tmp_path, variant, workload, fingerprint, nbytes):
    name = bench.traffic_record(workload, variant)
    with open(tmp_path / "profiles" / name, "w") as f:
        json.dump({"workload": workload, "kernel_sources": fingerprint, "dram_bytes_per_launch": nbytes}, f)


def test_traffic_record_follows_the_sources(tmp_path, monkeypatch):
    csrc = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("qwen3_full", "mean") is None              # no record
    fp = bench.score_kernel_fingerprint("mean")
    _record(tmp_path, "mean", "qwen3_full", fp, 12345)
    assert bench.ncu_traffic("qwen3_full", "mean") == 12345
    assert bench.ncu_traffic("qwen3_layer", "mean") is None             # another workload
    # a source the scorer is built from changes: the record no longer applies
    with open(csrc / "score.cuh", "a") as f:
        f.write("\n")
    assert bench.score_kernel_fingerprint("mean") != fp
    assert bench.ncu_traffic("qwen3_full", "mean") is None


def test_paged_records_are_kept_per_scorer(tmp_path, monkeypatch):
    """The paged workload has a record for the folded scorer and one for the
    max scorer; neither stands in for the other."""
    _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("qwen25_paged", "mean") != bench.traffic_record("qwen25_paged", "max")
    _record(tmp_path, "max", "qwen25_paged", bench.score_kernel_fingerprint("max"), 777)
    assert bench.ncu_traffic("qwen25_paged", "max") == 777
    assert bench.ncu_traffic("qwen25_paged", "mean") is None


def test_fingerprints_cover_each_scorers_sources(tmp_path, monkeypatch):
    csrc = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    before = {v: bench.score_kernel_fingerprint(v) for v in ("mean", "max", "pos")}
    with open(csrc / "score_pos_tma.cuh", "a") as f:      # only the distance scorer is built from it
        f.write("\n")
    after = {v: bench.score_kernel_fingerprint(v) for v in ("mean", "max", "pos")}
    assert after["mean"] == before["mean"] and after["max"] == before["max"]
    assert after["pos"] != before["pos"]
    with open(csrc / "common.cuh", "a") as f:             # every scorer includes it
        f.write("\n")
    assert all(bench.score_kernel_fingerprint(v) != after[v] for v in ("mean", "max", "pos"))


def test_gpus_flag_relaunches_one_process_per_gpu(monkeypatch):
    """`bench.py --gpus N` started by hand runs itself under torch.distributed.run
    with N processes and a loopback rendezvous, passing its own arguments on."""
    seen = {}

    def fake_call(cmd, timeout=None):
        seen["cmd"], seen["timeout"] = cmd, timeout
        return 0

    monkeypatch.setattr(bench.subprocess, "call", fake_call)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4", "--steps", "7", "--warmup", "3"])
    try:
        bench.main()
    except SystemExit as e:
        assert e.code == 0
    cmd = seen["cmd"]
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-6:] == ["--gpus", "4", "--steps", "7", "--warmup", "3"]
    assert cmd[-7].endswith("bench.py") and seen["timeout"] > 0


def test_bench_functions_read_only_names_they_can_see():
    """Every name a top-level function of bench.py reads is bound in it (or in
    a function nested in it), at module level, or is a builtin: the GPU legs
    cannot run here, so a stale name in one of them would only show on a GPU."""
    import ast
    import builtins
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    module = set(dir(builtins)) | {"__file__"}
    for node in tree.body:
        for n in ast.walk(node) if isinstance(node, (ast.Assign, ast.AnnAssign, ast.Import, ast.ImportFrom)) else []:
            if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Store):
                module.add(n.id)
            elif isinstance(n, ast.alias):
                module.add((n.asname or n.name).split(".")[0])
        if isinstance(node, (ast.FunctionDef, ast.ClassDef)):
            module.add(node.name)
    missing = []
    for fn in (n for n in tree.body if isinstance(n, ast.FunctionDef)):
        seen = set(module)
        for n in ast.walk(fn):
            if isinstance(n, ast.Name) and not isinstance(n.ctx, ast.Load):
                seen.add(n.id)
            elif isinstance(n, (ast.arg, ast.FunctionDef)):
                seen.add(n.arg if isinstance(n, ast.arg) else n.name)
            elif isinstance(n, ast.alias):
                seen.add((n.asname or n.name).split(".")[0])
            elif isinstance(n, ast.ExceptHandler) and n.name:
                seen.add(n.name)
        missing += [(fn.name, n.lineno, n.id) for n in ast.walk(fn)
                    if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load) and n.id not in seen]
    assert not missing, missing


def test_flush_writes_then_reads_the_whole_buffer():
    buf = torch.zeros(1000, dtype=torch.int32)
    sink = torch.zeros((), dtype=torch.int64)
    bench.flush_l2(buf, sink)
    assert int(sink) == 1000 and bool((buf == 1).all())
