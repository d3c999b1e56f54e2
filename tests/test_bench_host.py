"""Host-side logic of bench.py, on the CPU.

Covers the algorithmic FLOP count of every workload definition, the reader of
the nvidia-smi clock samples (which decides whether a timed run is kept), the
lookup of the measured peaks, and the gate that lets a stored ncu traffic
figure into the bench line only while the kernel sources are unchanged.
"""
import glob
import json
import os

import pytest

import bench
from rib_inputs import get_workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# GFLOP per layer, worked out from the shapes alone (units = B * windows *
# heads; per unit 2 N^2 (d_qk + d_v) forward and 2 N^2 (3 d_qk + 2 d_v)
# backward with d_qk = 48, d_v = 32, N = M^2).
@pytest.mark.parametrize("name,layer,units,fwd_gflop,bwd_gflop", [
    ("tiny", 0, 48, 0.503, 1.309),
    ("w32", 0, 384, 64.42, 167.5),
    ("cyclic", 0, 6912, 72.48, 188.4),
    ("cyclic", 1, 1728, 289.9, 753.8),
    ("cyclic", 2, 432, 1159.6, 3015.1),
    ("w96train", 0, 96, 1304.6, 3392.0),
    ("w96infer", 7, 144, 1956.9, 5088.0),
])
def test_flops_per_layer(name, layer, units, fwd_gflop, bwd_gflop):
    w = get_workload(name)
    assert w.units(layer) == units
    f, b = bench.flops(w, layer)
    assert f / 1e9 == pytest.approx(fwd_gflop, rel=1e-3)
    assert b / 1e9 == pytest.approx(bwd_gflop, rel=1e-3)


def test_inference_workload_total():
    # twelve 96x96 layers of 144 units: about 23.5 TFLOP per forward pass
    w = get_workload("w96infer")
    total = sum(bench.flops(w, l)[0] for l in range(w.layers))
    assert total / 1e12 == pytest.approx(23.483, rel=1e-3)
    assert w.tokens() == 576 * 384


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


class _FakeThread:
    def join(self, timeout=None):
        pass


def _sampler(lines):
    cs = bench.ClockSampler("0")
    cs.proc, cs.t, cs.lines = _FakeProc(), _FakeThread(), list(lines)
    return cs


def test_clock_samples_median_max_and_reasons():
    na = "Not Active"
    lines = [
        f"1965, 1965, 950.1, 0x0000000000000000, {na}, {na}, {na}, {na}",
        f"1905, 1965, 998.4, 0x0000000000000004, {na}, {na}, {na}, Active",
        f"1965, 1965, 991.0, 0x0000000000000004, {na}, {na}, {na}, Active",
        "garbage line",
        f"[N/A], 1965, 900.0, 0x0, {na}, {na}, {na}, {na}",
    ]
    r = _sampler(lines).stop()
    assert r["sm_mhz"] == 1965.0
    assert r["sm_max_mhz"] == 1965.0
    assert r["samples"] == 3
    assert r["power_w_max"] == pytest.approx(998.4)
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_samples_report_thermal_slowdown():
    na = "Not Active"
    r = _sampler([f"1500, 1965, 700.0, 0x40, {na}, Active, {na}, {na}"]).stop()
    assert r["reasons"] == ["hw_thermal_slowdown"]
    assert r["sm_mhz"] == 1500.0


def test_clock_samples_absent():
    assert _sampler([]).stop()["reasons"] == ["no samples"]
    cs = bench.ClockSampler("0")
    assert cs.stop()["reasons"] == ["nvidia-smi unavailable"]


def test_peaks_measured_and_fallback(monkeypatch, tmp_path):
    d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    p = bench.peaks()
    assert p["source"] == "measured"
    assert p["hbm_gbs"] == d["hbm_gbs"]
    assert p["bf16_tflops_sustained"] == d["bf16_tflops_sustained"]
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f = bench.peaks()
    assert f["source"] == "fallback"
    assert (f["hbm_gbs"], f["bf16_tflops"]) == (6650.0, 1590.0)


def test_stored_traffic_follows_the_kernel_sources(monkeypatch, tmp_path):
    csrc = tmp_path / "windowed_attention_implicit_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cuh").write_text("// kernel v1\n")
    (csrc / "notes.txt").write_text("not a source\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash()
    rec = {"kernel": "k", "workload": "w", "source_hash": h, "dram_bytes_per_launch": 1234}
    (tmp_path / "profiles" / "k_w.traffic.json").write_text(json.dumps(rec))
    assert bench.stored_traffic("k", "w") == 1234
    assert bench.stored_traffic("k", "other") is None
    (csrc / "notes.txt").write_text("edited, still not a source\n")
    assert bench.stored_traffic("k", "w") == 1234
    (csrc / "k.cuh").write_text("// kernel v2\n")
    assert bench.kernel_source_hash() != h
    assert bench.stored_traffic("k", "w") is None


def test_stored_traffic_of_a_listed_kernel_follows_its_own_sources(monkeypatch, tmp_path):
    csrc = tmp_path / "windowed_attention_implicit_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cuh").write_text("// kernel a v1\n")
    (csrc / "common.cuh").write_text("// shared v1\n")
    (csrc / "b.cuh").write_text("// kernel b v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", {"ka": ("a.cuh", "common.cuh")})
    h = bench.kernel_source_hash("ka")
    assert h != bench.kernel_source_hash()          # a subset of the sources
    rec = {"kernel": "ka", "workload": "w", "source_hash": h, "dram_bytes_per_launch": 99}
    (tmp_path / "profiles" / "ka_w.traffic.json").write_text(json.dumps(rec))
    assert bench.stored_traffic("ka", "w") == 99
    (csrc / "b.cuh").write_text("// kernel b v2\n")   # another kernel's source
    assert bench.stored_traffic("ka", "w") == 99
    (csrc / "common.cuh").write_text("// shared v2\n")  # one of its own
    assert bench.stored_traffic("ka", "w") is None


def test_committed_traffic_records_match_the_current_sources():
    """Every committed record was taken from the sources now in the tree
    (a stale record is nulled by the bench; this keeps the committed ones
    current)."""
    for p in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.traffic.json"))):
        d = json.load(open(p))
        assert d["source_hash"] == bench.kernel_source_hash(d["kernel"]), os.path.basename(p)


def test_committed_traffic_records_are_well_formed():
    recs = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.traffic.json")))
    assert recs
    for p in recs:
        d = json.load(open(p))
        assert os.path.basename(p) == f"{d['kernel']}_{d['workload']}.traffic.json"
        assert d["dram_bytes_read"] > 0 and d["dram_bytes_write"] >= 0
        assert d["dram_bytes_per_launch"] == d["dram_bytes_read"] + d["dram_bytes_write"]
        assert len(d["source_hash"]) == 16
        assert "--clock-control none" in d["command"] and d["command"].startswith("ncu ")


# ---------------------------------------------------------------- ranks

def test_world_plan():
    assert bench.world_plan(1, {}) == "run"
    assert bench.world_plan(4, {}) == "relaunch"
    assert bench.world_plan(2, {"WORLD_SIZE": "2"}) == "run"
    assert bench.world_plan(1, {"WORLD_SIZE": "1"}) == "run"
    with pytest.raises(ValueError, match="WORLD_SIZE=2"):
        bench.world_plan(8, {"WORLD_SIZE": "2"})
    with pytest.raises(ValueError, match="WORLD_SIZE=4"):
        bench.world_plan(1, {"WORLD_SIZE": "4"})
    with pytest.raises(ValueError):
        bench.world_plan(0, {})


def test_relaunch_command_starts_n_ranks_of_this_script():
    cmd = bench.relaunch_cmd(8, ["--gpus", "8", "--steps", "3"], 29511)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=8" in cmd and "--nnodes=1" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[cmd.index("--master-port") + 1] == "29511"
    assert cmd[-4:] == ["--gpus", "8", "--steps", "3"]
    assert os.path.samefile(cmd[-5], os.path.join(ROOT, "bench.py"))


def test_both_arms_share_one_config_object():
    w = get_workload("w96train")
    c = bench.bench_config(w, 2)
    assert c["global_batch"] == 8 and c["parallelism"] == "dp2"
    assert c["map"] == [192, 192] and (c["window"], c["shift"]) == (96, 48)
    assert (c["heads"], c["head_dim"], c["rank"]) == (6, 32, 16)
    assert c["workload"].startswith("w96train:")


def test_roofline_divides_by_the_burst_peak():
    pk = {"bf16_tflops": 1665.3, "bf16_tflops_sustained": 1404.1, "source": "measured"}
    e = bench.roofline_entry("attn_bwd_kernel", 3.392e12, 4.655, pk)
    assert e["achieved"] == pytest.approx(3.392e12 / 4.655e-3 / 1e12)
    assert e["peak"] == 1665.3
    assert e["frac"] == pytest.approx(0.4376, abs=1e-4)
    assert e["frac_of_sustained"] == pytest.approx(e["achieved"] / 1404.1)
    assert "burst" in e["peak_source"]


def _max_over_ranks_worker(rank, world, port, q):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        q.put((rank, bench.max_over_ranks([3.5, 7.25][rank], "cpu")))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = bench.free_port()
    ps = [ctx.Process(target=_max_over_ranks_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    got = dict(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 7.25, 1: 7.25}
