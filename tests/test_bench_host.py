"""Host-side logic of the bench on the CPU:
- algorithmic byte formulas;
- clock parsing and the rejection rules;
- max-over-ranks timing across 2 gloo ranks;
- the reference arm's JSON line, and rank > 0 exiting quietly."""
import json
import os
import subprocess
import sys

import torch.multiprocessing as mp

from combine_top_group_b200 import metrics
from combine_top_group_b200 import workloads as wl
from conftest import ROOT


def test_byte_formulas_prefill():
    w = wl.WORKLOADS["prefill"]
    M = w.N * w.K
    d = metrics.dispatch_bytes(w, M)
    c = metrics.combine_bytes(w, M)
    # dominant terms: read N rows once, write M rows (bf16) / read M rows, write N rows
    assert d == w.N * w.H * 2 + M * w.H * 2 + w.N * w.K * 8 + M * 8
    assert c == M * w.H * 2 + w.N * w.H * 2 + w.N * w.K * 8
    assert 4.22e9 < d < 4.24e9 and 4.22e9 < c < 4.24e9
    assert metrics.layout_bytes(w) == w.N * w.E * 4 + w.N * w.K * 12 + w.N * w.R


def test_byte_formulas_fp8():
    w = wl.WORKLOADS["large"]
    M = w.N * w.K
    d = metrics.dispatch_bytes(w, M)
    assert d == w.N * w.H * 2 + w.N * w.K * 8 + M * w.H + M * (w.H // 128) * 4 + M * 8
    assert metrics.combine_bytes(w, M, fused_fp8=True) == M * w.H + M * 56 * 4 + w.N * w.K * 8 + w.N * w.H * 2


CSV = """index, clocks.current.sm [MHz], clocks.max.sm [MHz], power.draw [W], clocks_event_reasons.active, clocks_event_reasons.hw_slowdown, clocks_event_reasons.hw_thermal_slowdown, clocks_event_reasons.sw_thermal_slowdown, clocks_event_reasons.sw_power_cap
0, 1965 MHz, 1965 MHz, 700.1 W, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active
0, 1800 MHz, 1965 MHz, 990.0 W, 0x0000000000000004, Not Active, Not Active, Not Active, Active
0, 1900 MHz, 1965 MHz, 900.0 W, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active
"""


def test_parse_clocks_and_rules():
    c = metrics.parse_clocks(CSV.replace("clocks.current.sm", "clocks.sm"))
    assert c["sm_mhz"] == 1900 and c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]
    assert metrics.clocks_rejected(c) is None
    assert "throttled" in metrics.clocks_rejected({"sm_mhz": 1900, "sm_max_mhz": 1965, "reasons": ["hw_slowdown"]})
    assert "clock lock" in metrics.clocks_rejected({"sm_mhz": 800, "sm_max_mhz": 1965, "reasons": []})
    s = metrics.summarize_nvml([(1900, 1965, 800.0, 0x4), (1700, 1965, None, 0x40)], metrics.ClockSampler._BITS)
    assert s["power_w_max"] == 800.0
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"] and s["sm_mhz"] == 1800


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    got = metrics.max_over_ranks([1.0 + rank, 5.0 - rank])
    q.put((rank, got))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [2.0, 5.0]


def bench_host_cores():
    import bench
    return bench.host_cores()


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["cores"] == bench_host_cores() and line["cpu_baseline"]["host"]["nproc"] >= 1
    # both arms print the same metric, so their values compare directly
    import bench
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True
    # the line names the sample it timed
    assert line["config"]["sample_tokens_per_rank"] == min(wl.WORKLOADS["tiny"].T, bench.ORACLE_SAMPLE_T)


def test_one_core_pin_is_restored():
    import bench
    if not hasattr(os, "sched_getaffinity"):
        return
    before = os.sched_getaffinity(0)
    with bench.OneCore():
        assert len(os.sched_getaffinity(0)) == 1
    assert os.sched_getaffinity(0) == before


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


NCU_CSV = '''==PROF== Connected to process 1
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","1","python3.12","h","void unnamed>::layout_kernel<8>(unnamed>::LayoutParams)","1","7","(256, 1, 1)","(296, 1, 1)","0","10.0","m","dram__bytes_read.sum","Mbyte","33.63"
"0","1","python3.12","h","void unnamed>::layout_kernel<8>(unnamed>::LayoutParams)","1","7","(256, 1, 1)","(296, 1, 1)","0","10.0","m","dram__bytes_write.sum","byte","0"
"1","1","python3.12","h","void unnamed>::dispatch_bf16_kernel<1>(unnamed>::DispatchParams)","1","7","(448, 1, 1)","(32768, 1, 1)","0","10.0","m","dram__bytes_read.sum","byte","472,184,064"
"1","1","python3.12","h","void unnamed>::dispatch_bf16_kernel<1>(unnamed>::DispatchParams)","1","7","(448, 1, 1)","(32768, 1, 1)","0","10.0","m","dram__bytes_write.sum","byte","3698034176"
"2","1","python3.12","h","void unnamed>::combine_dedup_kernel(unnamed>::P)","1","7","(128, 1, 1)","(10, 1, 1)","0","10.0","m","dram__bytes_read.sum","byte","5"
"3","1","python3.12","h","void unnamed>::combine_bf16_kernel<1>(unnamed>::CombineParams)","1","7","(128, 1, 1)","(32768, 1, 1)","0","10.0","m","dram__bytes_read.sum","Gbyte","3.76"
"3","1","python3.12","h","void unnamed>::combine_bf16_kernel<1>(unnamed>::CombineParams)","1","7","(128, 1, 1)","(32768, 1, 1)","0","10.0","m","dram__bytes_write.sum","Mbyte","458.6"
'''


def test_ncu_traffic_parse_and_hash(tmp_path, monkeypatch):
    t = metrics.traffic_from_ncu(NCU_CSV)
    assert set(t) == {"layout", "dispatch", "combine"}  # combine_dedup is not the combine kernel
    assert t["layout"]["dram_bytes_per_launch"] == 33_630_000
    assert t["dispatch"]["dram_read"] == 472_184_064 and t["dispatch"]["dram_write"] == 3_698_034_176
    assert t["combine"]["dram_bytes_per_launch"] == 3_760_000_000 + 458_600_000
    # per-kernel hashes: each kernel's figure is tied to its own sources only
    assert t["dispatch"]["source_hash"] == metrics.source_hash("dispatch")
    assert len({metrics.source_hash(k) for k in ("layout", "dispatch", "combine")}) == 3
    f = tmp_path / "traffic.json"
    c = tmp_path / "ncu.csv"
    c.write_text(NCU_CSV)
    monkeypatch.setattr(metrics, "TRAFFIC_FILE", str(f))
    # a capture at 1024 tokens per rank scales by 4096 / 1024 to the prefill workload
    ent = metrics.record_traffic(str(c), "prefill", "dispatch", "ncu ... -k regex:dispatch -c 1 ...", 1024)
    assert ent["scale_to_workload"] == 4.0
    assert metrics.stored_traffic("dispatch", "prefill") == 4 * (472_184_064 + 3_698_034_176)
    assert metrics.stored_traffic("combine", "prefill") is None  # not recorded
    assert metrics.stored_traffic("dispatch", "large") is None
    metrics.record_traffic(str(c), "prefill", "combine", "ncu ...", 1024)
    data = json.loads(f.read_text())
    data["prefill"]["combine"]["source_hash"] = "0" * 16  # captured from other sources
    f.write_text(json.dumps(data))
    assert metrics.stored_traffic("combine", "prefill") is None
    assert metrics.stored_traffic("dispatch", "prefill") is not None


def test_ep_workload_one_rank_per_gpu():
    """--gpus N runs the workload with R = N ranks, each keeping the
    workload's T tokens (weak scaling); E must split evenly over the ranks."""
    import pytest

    import bench
    w = wl.WORKLOADS["prefill"]
    for n in (1, 2, 4, 8):
        e = bench.ep_workload(w, n)
        assert (e.R, e.T, e.E, e.K, e.H, e.G, e.KG) == (n, w.T, w.E, w.K, w.H, w.G, w.KG)
        assert e.L == w.E // n
    with pytest.raises(SystemExit):
        bench.ep_workload(w, 3)  # 256 experts do not split over 3 ranks
    with pytest.raises(SystemExit):
        bench.ep_workload(wl.WORKLOADS["decode_ll"], 2)  # the low-latency layout has no per-GPU path
    a = bench.parse_args(["--gpus", "8", "--replicas"])
    assert a.replicas and not a.one_rank_per_gpu
