"""Host-side logic of bench.py that needs no GPU: the multi-rank timing
reduction over a world-2 gloo group, the reference arm's rank handling and
JSON line, and the parsing of clock samples."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # every rank times something different; all must report the slowest
        got = bench._max_over_ranks(1.5 + 2.0 * rank, world)
        bench._barrier(world)
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
            json.dump({"max": got}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_world2_gloo(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        with open(tmp_path / ("rank%d.json" % r)) as f:
            assert json.load(f)["max"] == 1.5 + 2.0 * (world - 1)


def _run_bench(args, env_extra, timeout=600):
    env = dict(os.environ)
    env.update(env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, env=env, timeout=timeout)


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"],
                   {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_line():
    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "3"],
                   {"RANK": "0", "LOCAL_RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "Mtok/s"
    assert line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["warmup"] == 3
    assert line["config"] == bench._config(8192, 96, 128)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "Mtok/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_clock_summary_parsing(tmp_path):
    rows = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1830, 1965, 985.3, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "0, [N/A], 1965, 10, 0, Not Active, Not Active, Not Active, Not Active",
    ]
    path = tmp_path / "clk.csv"
    path.write_text("\n".join(rows) + "\n")
    cs = bench.ClockSampler(0)
    cs.path = str(path)
    s = cs.summary()
    assert s["sm_mhz"] == 1830.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    assert not path.exists()        # the temporary file is removed


def test_default_run_on_cpu_fails_loudly():
    """Without a GPU the product arm must not fall back to anything."""
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    r = _run_bench(["--steps", "1", "--warmup", "3"], {"WORLD_SIZE": "1"}, timeout=300)
    assert r.returncode != 0
    assert not any(ln.startswith("{") for ln in r.stdout.splitlines())


def test_traffic_record_round_trip(tmp_path, monkeypatch):
    """bench.py --record-traffic reads an ncu CSV log, keeps the prefill
    kernel's DRAM counters (converting the units), keys them by the kernel
    source hash, and the roofline reads them back only while that hash holds."""
    import bench
    csv_text = (
        '"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream",'
        '"Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit",'
        '"Metric Value"\n'
        '"0","1","python","h","void kda::decode_step_kernel","1","7","(256,1,1)","(9,1,1)","0",'
        '"10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","5.00"\n'
        '"1","1","python","h","prefill::chunk_fwd_sm100_kernel<false>(...)","1","7","(512,1,1)",'
        '"(96,1,1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte",'
        '"809.60"\n'
        '"1","1","python","h","prefill::chunk_fwd_sm100_kernel<false>(...)","1","7","(512,1,1)",'
        '"(96,1,1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","Kbyte",'
        '"186,400.00"\n')
    log = tmp_path / "k3.csv"
    log.write_text(csv_text)
    rec_path = tmp_path / "rec.json"
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(rec_path))
    bench.record_traffic(str(log), "ncu ... (test)")
    assert bench._measured_traffic() == pytest.approx(809.6e6 + 186.4e6)
    monkeypatch.setattr(bench, "_prefill_source_hash", lambda: "0" * 16)
    assert bench._measured_traffic() is None


def test_layer_rows_report_and_isolate_failures(monkeypatch):
    """The bench's rows for the prologue, the gated prefill and the softplus
    variant: a measured row carries its time, throughput and roofline
    fraction; a row whose call raises, or whose kernel reports a bad status,
    carries the error instead, and the others are still measured."""
    import bench

    class FakeBinding:
        KDA_OK = 0
        status = [0, 5]          # OK after the prologue, a timeout after the gated call

        def kda_stream_status(self, stream=None):
            return self.status.pop(0)

        def kda_status_string(self, st):
            return "a kernel's bounded wait ran out"

    def prologue(dev, stream, binding, inputs):
        return 0.25, 1_000_000_000, 8192, 96

    def gated(dev, stream, binding, inputs):
        return 0.8, 1_200_000_000, 8192, 96

    def softplus(dev, stream, binding, inputs):
        raise RuntimeError("no such kernel")

    monkeypatch.setattr(bench, "_prologue_local", prologue)
    monkeypatch.setattr(bench, "_gated_local", gated)
    monkeypatch.setattr(bench, "_softplus_local", softplus)
    rows = bench._measure_layer_rows("cpu", None, 1, 8000.0, 0.7, FakeBinding(), None)
    p = rows["prologue_k3"]
    assert p["ms"] == 0.25 and p["hbm_gbs"] == pytest.approx(4000.0)
    assert p["frac_of_peak"] == pytest.approx(0.5)
    assert p["Mtok_s"] == pytest.approx(8192 / 0.25e-3 / 1e6)
    assert rows["gated_k3"] == {"error": "kernel status: a kernel's bounded wait ran out"}
    assert rows["softplus_2k"]["error"].startswith("RuntimeError: no such kernel")


def test_gated_row_reports_its_cost_over_the_plain_launch(monkeypatch):
    import bench

    class FakeBinding:
        KDA_OK = 0

        def kda_stream_status(self, stream=None):
            return 0

    for name in ("_prologue_local", "_gated_local", "_softplus_local"):
        monkeypatch.setattr(bench, name, lambda *a: (0.77, 10**9, 8192, 96))
    rows = bench._measure_layer_rows("cpu", None, 1, 8000.0, 0.7, FakeBinding(), None)
    assert rows["gated_k3"]["cost_over_plain"] == pytest.approx(0.1)
    assert "cost_over_plain" not in rows["prologue_k3"]
    json.dumps(rows)


class _OkBinding:
    KDA_OK = 0

    def kda_stream_status(self, stream=None):
        return 0


def _layer_rank_main(rank, world, port, out_dir):
    """One rank of the layer-row measurement: rank 0's gated call fails, every
    other call succeeds with a rank-dependent time."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        def ok(*a):
            return 0.5 + rank, 10**9, 8192, 96

        def gated(*a):
            if rank == 0:
                raise RuntimeError("launch failed")
            return ok()

        bench._prologue_local, bench._gated_local, bench._softplus_local = ok, gated, ok
        rows = bench._measure_layer_rows("cpu", None, world, 8000.0, 0.7, _OkBinding(), None)
        with open(os.path.join(out_dir, "layer%d.json" % rank), "w") as f:
            json.dump(rows, f)
    finally:
        dist.destroy_process_group()


def test_layer_rows_world2_gloo_one_rank_fails(tmp_path):
    """Every rank takes the same collective steps: a call that fails on one
    rank ends as an error row on all ranks (no rank waits for good), and the
    rows that succeed everywhere report the slowest rank's time."""
    world = 2
    mp.start_processes(_layer_rank_main, args=(world, _free_port(), str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        with open(tmp_path / ("layer%d.json" % r)) as f:
            rows = json.load(f)
        assert rows["prologue_k3"]["ms"] == 1.5 and rows["softplus_2k"]["ms"] == 1.5
        assert "error" in rows["gated_k3"]
    with open(tmp_path / "layer1.json") as f:
        assert json.load(f)["gated_k3"] == {"error": "failed on another rank"}


def test_layer_row_calls_bind_to_the_binding(monkeypatch):
    """The three row measurements call the real binding's functions with
    arguments that bind to their signatures, tensors of the shapes the
    binding checks, and the keyword stream: checked on small shapes on the
    CPU with a stand-in that records each call instead of launching."""
    import inspect
    import bench
    from gated_delta_rule_60_b200 import binding as real, inputs

    calls = []

    class Recorder:
        KDA_OK = 0

        def __getattr__(self, name):
            fn = getattr(real, name)

            def record(*a, **kw):
                bound = inspect.signature(fn).bind(*a, **kw)
                calls.append((name, bound.arguments))
            return record

    monkeypatch.setattr(bench, "LAYER_ROW_SHAPES", {"prologue_k3": (40, 3, 16),
                                                    "gated_k3": (40, 3, 16),
                                                    "softplus_2k": (24, 2, 32)})
    monkeypatch.setattr(bench, "_events_ms", lambda stream, fn, w, s: (fn(), 1.0)[1])
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    stream = object()
    for fn in (bench._prologue_local, bench._gated_local, bench._softplus_local):
        fn("cpu", stream, Recorder(), inputs)
    names = [c[0] for c in calls]
    assert names == ["kda_prologue", "kda_chunk_fwd_gated", "kda_chunk_fwd_softplus"]
    pro, gated, soft = (c[1] for c in calls)
    assert pro["xq"].shape == (40, 3, 16) and pro["wq"].shape == (3, 16, 4)
    assert pro["beta_raw"].shape == (40, 3) and pro["cu_seqlens"].tolist() == [0, 40]
    assert gated["z"].shape == gated["v"].shape == gated["o"].shape == (40, 3, 16)
    assert gated["hT"].shape == (1, 3, 16, 16) and gated["h0"] is None
    assert soft["h0"].shape == soft["hT"].shape == (1, 2, 32, 32)
    for args in (pro, gated, soft):
        assert args["stream"] is stream
        assert all(t.dtype in (torch.bfloat16, torch.float32, torch.int32)
                   for t in args.values() if isinstance(t, torch.Tensor))
