"""Host logic of the benchmark on CPU: the replica (data-parallel) layout with two ranks
over gloo.  Each rank draws its own batch, the timing reduction takes the max over
ranks, and the whole-job value counts every rank's tokens.  Also the traffic lookup, the
per-kernel rooflines, and the reference arm's JSON line."""
import json
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from hybrid_softmax_linear_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        out[rank] = bench.reduce_max(local_ms, world, torch.device("cpu"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_gloo_world_size_2():
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0] == out[1] == 15.0


def test_whole_job_value_counts_every_replica():
    assert bench.whole_job_value(1, 90720, 50.0) == 90720 / 0.05
    assert bench.whole_job_value(4, 90720, 50.0) == 4 * 90720 / 0.05


def test_replicas_draw_distinct_batches():
    a = synth.workload_inputs(1, rank=0)
    b = synth.workload_inputs(1, rank=1)
    c = synth.workload_inputs(1, rank=0)
    assert not np.array_equal(a["q"], b["q"])
    for n in a:
        np.testing.assert_array_equal(a[n], c[n])      # deterministic per rank


def test_softmax_flop_count_matches_brute_force():
    s = synth.Shape(12, 7, 2, 3, 2, 32)
    from oracle import vdn_oracle as vo
    M = vo.frame_mask(s.frames, s.chunk_frames)
    keys = sum(s.tokens_per_frame * (s.text_tokens + s.tokens_per_frame * int((M[f] == vo.SOFT).sum()))
               for f in range(s.frames))
    assert bench.softmax_flops(s) == 4.0 * s.head_dim * s.heads * keys


def test_captured_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed capture only while the kernel source is the
    one captured, scaled by query rows x heads."""
    import hashlib
    src = tmp_path / "k.cu"
    src.write_text("kernel source\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    cap = tmp_path / "cap.json"
    cap.write_text(json.dumps({"source_sha256": sha, "bf16": {"bytes": 1000, "units": 10}}))
    monkeypatch.setattr(bench, "SOFTMAX_SRC", str(src))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(cap))
    shape = synth.Shape(2, 5, 1, 0, 2, 32)                     # 10 rows x 2 heads = 20 units
    t, how = bench.captured_traffic(shape, fp8=False)
    assert t == 2000.0 and "scaled" in how
    assert bench.captured_traffic(shape, fp8=True)[0] is None  # no e4m3 entry
    src.write_text("changed\n")
    assert bench.captured_traffic(shape, fp8=False)[0] is None



def test_kernel_rooflines_use_the_algorithmic_work():
    """Per-kernel rates divide the stated algorithmic work by the live time per call."""
    shape = synth.CONFIGS[2].shape
    work = bench.kernel_work(shape, "elu1", fp8=False)
    Nv, HD = shape.n_video, shape.heads * shape.head_dim
    assert work["read_tc"] == ("hbm", 2.0 * Nv * HD * 2)
    assert work["softmax_tc"] == ("tensor", bench.softmax_flops(shape))
    peaks = {"bf16_tflops": 1000.0, "bf16_tflops_sustained": 800.0, "hbm_gbs": 5000.0}
    prof = {"read_tc": (2.0, 4), "softmax_tc": (10.0, 2), "tables": (0.1, 2)}
    k = bench.kernel_rooflines(prof, 2, shape, "elu1", False, peaks, 1.0)
    assert set(k) == {"read_tc", "softmax_tc"}                 # no work figure for the tables
    gbs = work["read_tc"][1] / 0.5e-3 / 1e9
    assert abs(k["read_tc"]["gb_per_s"] - round(gbs, 1)) < 0.11
    tf = work["softmax_tc"][1] / 5e-3 / 1e12
    assert abs(k["softmax_tc"]["frac_of_sustained"] - round(tf / 800.0, 3)) < 1e-3
    assert "fp8_quant" in bench.kernel_work(shape, "delta", fp8=True)


def _bench_reference(env_extra):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config", "1",
                        "--steps", "2", "--warmup", "1"], cwd=root, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_reference_arm_prints_the_contract_line_on_rank_0_only():
    """--impl reference times the CPU oracle on rank 0 and prints one JSON line with the
    arm's keys; another rank of a multi-rank launch exits 0 without work."""
    lines = _bench_reference({"RANK": "0", "WORLD_SIZE": "1"})
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT and d["steps"] == 2 and d["warmup"] == 1
    assert d["config"]["workload"] == synth.CONFIGS[1].name
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert _bench_reference({"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_clock_sampler_summarises_only_the_timed_region(monkeypatch):
    """The sampler takes one NVML reading before the timed region starts (the first reads
    can outlast a short region) and leaves it out of the summary; reasons decode from the
    event-reason bits.  NVML is a fake here: nothing on a GPU is read or set."""
    import sys
    import time
    import types
    fake = types.ModuleType("pynvml")
    fake.NVML_CLOCK_SM = 0
    fake.nvmlInit = lambda: None
    fake.nvmlDeviceGetHandleByUUID = lambda uuid: object()
    clock = iter([400] + [1900] * 1000)  # an idle reading first, then clocks under load

    def get_clock(h, kind):
        time.sleep(0.03)
        return next(clock)
    fake.nvmlDeviceGetClockInfo = get_clock
    fake.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4  # sw_power_cap
    fake.nvmlDeviceGetPowerUsage = lambda h: 700_000
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: types.SimpleNamespace(uuid="0"))
    sampler = bench.ClockSampler(0)
    assert sampler.skip >= 1
    time.sleep(0.2)
    got = sampler.stop()
    assert got["source"] == "nvml" and got["samples"] >= 2
    assert got["sm_mhz"] == 1900 and got["sm_max_mhz"] == 1965
    assert got["reasons"] == ["sw_power_cap"] and got["power_w_max"] == 700.0


def test_linear_bwd_only_refuses_configurations_without_an_elu1_bf16_branch(monkeypatch):
    """--linear-bwd-only times the elu+1 backward; a delta-rule or e4m3 configuration is
    refused on the host before any device work."""
    import sys
    monkeypatch.setattr(sys, "argv", ["bench.py", "--linear-bwd-only", "--config", "5"])
    try:
        bench.main()
    except SystemExit as e:
        assert "elu+1 bf16" in str(e.code)
    else:
        raise AssertionError("configuration 5 was accepted")


def test_backward_cpu_baseline_times_a_head_sample_of_the_oracle():
    """The backward leg's CPU baseline runs the float64 backward oracle on a head slice and
    scales by the head count; it reports the contract's keys."""
    w = synth.CONFIGS[1]
    inp = synth.workload_inputs(1)
    got = bench.oracle_bwd_sample(w.shape, inp, heads=1)
    assert got["kind"] == "oracle" and got["unit"] == bench.UNIT and got["cores"] >= 1
    assert got["value"] > 0 and f"1 of {w.shape.heads} heads" in got["sample"]
