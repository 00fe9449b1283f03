"""Host-side logic of bench.py on CPU: the roofline's DRAM traffic comes from a committed ncu summary
only while every source file that summary hashes is unchanged; otherwise it is reported as null."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import workloads as W  # noqa: E402

SUMMARY = "fwd_tc_kernel.drafter_s32k.txt"


def _copy_summary_and_sources(dst):
    src_summary = os.path.join(ROOT, "profiles", SUMMARY)
    lines = open(src_summary).read().splitlines()
    rels = [ln[len("source_sha256 "):].split(": ")[0] for ln in lines if ln.startswith("source_sha256 ")]
    assert rels, "the summary names the sources it was captured from"
    os.makedirs(os.path.join(dst, "profiles"))
    shutil.copy(src_summary, os.path.join(dst, "profiles", SUMMARY))
    for rel in rels:
        os.makedirs(os.path.dirname(os.path.join(dst, rel)), exist_ok=True)
        shutil.copy(os.path.join(ROOT, rel), os.path.join(dst, rel))
    traffic = int([ln for ln in lines if ln.startswith("traffic_bytes_per_launch:")][0].split(":")[1])
    return rels, traffic


def _write_hashes_of_current_sources(root, rels):
    # Make the copied summary describe the copied sources exactly as they are.
    import hashlib
    path = os.path.join(root, "profiles", SUMMARY)
    out = []
    for ln in open(path).read().splitlines():
        if ln.startswith("source_sha256 "):
            rel = ln[len("source_sha256 "):].split(": ")[0]
            ln = f"source_sha256 {rel}: " + hashlib.sha256(open(os.path.join(root, rel), "rb").read()).hexdigest()
        out.append(ln)
    open(path, "w").write("\n".join(out) + "\n")


def test_traffic_reported_while_sources_match(tmp_path, monkeypatch):
    rels, traffic = _copy_summary_and_sources(str(tmp_path))
    _write_hashes_of_current_sources(str(tmp_path), rels)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("fwd_tc_kernel", "drafter_s32k") == traffic > 0


def test_traffic_null_once_a_source_changed(tmp_path, monkeypatch):
    rels, _ = _copy_summary_and_sources(str(tmp_path))
    _write_hashes_of_current_sources(str(tmp_path), rels)
    with open(os.path.join(str(tmp_path), rels[-1]), "a") as f:
        f.write("\n// edited after the capture\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("fwd_tc_kernel", "drafter_s32k") is None


def test_traffic_follows_the_workload_definition(tmp_path, monkeypatch):
    # A summary pins the workload it was captured on (its dataclass repr): another run length, cost tile
    # or packing in the registry makes its traffic stale, whatever the source hashes say.
    import dataclasses
    rels, traffic = _copy_summary_and_sources(str(tmp_path))
    _write_hashes_of_current_sources(str(tmp_path), rels)
    path = os.path.join(str(tmp_path), "profiles", SUMMARY)
    lines = [ln for ln in open(path).read().splitlines() if not ln.startswith("workload: ")]
    open(path, "w").write("\n".join(lines + ["workload: " + repr(W.get("drafter_s32k"))]) + "\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("fwd_tc_kernel", "drafter_s32k") == traffic > 0
    changed = dataclasses.replace(W.get("drafter_s32k"), chunks_per_item=W.get("drafter_s32k").chunks_per_item + 1)
    monkeypatch.setitem(W.WORKLOADS, "drafter_s32k", changed)
    assert bench.profiled_traffic("fwd_tc_kernel", "drafter_s32k") is None


def test_traffic_null_without_a_summary(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("fwd_tc_kernel", "drafter_s32k") is None


def test_useful_flops_count_the_pairs_the_oracle_sees():
    # 4 d FLOP per (query row, visible key, query head) forward (QK^T and PV), 10 d backward, with the
    # visible keys taken from the oracle's own visibility rule, block by block.
    import workloads as W
    from tests._util import oracle_problem
    for w in (W.get("tiny_f32"), W.scaled(W.get("train_4x64k"), "flops", [3000, 2048], [3, 2], chunk=1024)):
        inp = W.make_inputs(w)
        p = oracle_problem(inp)
        pairs = 0
        for s, j, a in p.blocks():
            for h in range(p.Hq):
                keys, _ = p.visible(s, j, a, h // p.G)
                pairs += p.block * keys.shape[0]
        total, fwd = bench.useful_flops(inp, backward=True)
        assert fwd == 4 * p.d * pairs
        assert total == 14 * p.d * pairs
        assert bench.useful_flops(inp, backward=False) == (fwd, fwd)


def test_clock_reason_bits_are_nvmls():
    pynvml = __import__("pynvml")
    names = {"hw_slowdown": "HwSlowdown", "hw_thermal_slowdown": "HwThermalSlowdown",
             "sw_thermal_slowdown": "SwThermalSlowdown", "sw_power_cap": "SwPowerCap"}
    for name, bit in bench.ClockSampler.REASONS:
        assert bit == getattr(pynvml, "nvmlClocksEventReason" + names[name]), name


def test_clock_summary_of_samples():
    c = bench.ClockSampler(0)
    assert c.summary()["source"] == "none" and c.summary()["samples"] == 0
    c.samples = [(1965.0, 1965.0, 0x0), (1800.0, 1965.0, 0x4), (1700.0, 1965.0, 0x4 | 0x40)]
    s = c.summary()
    assert s["sm_mhz"] == 1800.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_oracle_planning_time_and_cpu_model():
    import workloads as W
    inp = W.make_inputs(W.get("tiny_f32"))
    r = bench.cpu_oracle_plan(inp, 4)
    assert r["items"] == 19 and r["workers"] == 4 and r["threads"] == 1
    assert r["cost_ms"] >= 0 and r["lpt_ms"] >= 0
    assert isinstance(bench.cpu_model(), str) and bench.cpu_model()


def test_timed_step_count_reaches_one_second():
    # Without --steps the timed region holds at least 1 s of steps (and at least 20 steps).
    assert bench.timed_step_count(15.0) == 67          # skewed_s256k-sized steps: 67 x 15 ms >= 1 s
    assert bench.timed_step_count(0.35) == 2858        # drafter-sized steps
    assert bench.timed_step_count(100.0) == 20         # long steps: the minimum count
    for ms in (0.01, 0.2, 3.3, 12.4, 49.9):
        n = bench.timed_step_count(ms)
        assert n >= 20 and n * ms >= 1000.0 and (n == 20 or (n - 1) * ms < 1000.0)


def test_traffic_only_for_the_registered_workload_and_plan():
    # An override of the run length, cost tile or packing, or the naive plan, moves other DRAM bytes than
    # the committed ncu summary of the workload holds: no traffic in that line.
    import argparse
    args = argparse.Namespace(workload="long_s128k", blocks_per_item=0, chunks_per_item=0, key_tile=0,
                              item_overhead=-1)
    w = bench.workload_of(args)
    assert w == W.get("long_s128k") and bench.traffic_applies(w, "lpt")
    assert not bench.traffic_applies(w, "naive")
    for k, v in (("chunks_per_item", w.chunks_per_item // 2), ("key_tile", w.key_tile // 2), ("blocks_per_item", 2)):
        w2 = bench.workload_of(argparse.Namespace(**{**vars(args), k: v}))
        assert getattr(w2, k) == v and not bench.traffic_applies(w2, "lpt")
    assert not bench.traffic_applies(W.get("tiny_f32"), "lpt")


def test_library_provenance_names_the_build():
    prov = bench.library_provenance()
    assert prov["matches_sources"] is True and len(prov["build_id"]) == 16
