"""Host-side checks of bench.py that need no GPU: the multi-rank timing
aggregation over a two-rank gloo group, and the reference arm (the CPU
oracle) printing its JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [2.0, 3.5][rank]                       # ms per step on this rank
        ms = bench.max_over_ranks(mine)
        out[rank] = (ms, bench.job_throughput(128, world, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    for rank in (0, 1):
        ms, tput = res[rank]
        assert ms == 3.5                              # the slowest rank's time
        assert tput == pytest.approx(2 * 128 / 3.5e-3)   # all ranks' tokens


def test_single_process_aggregation():
    assert bench.max_over_ranks(1.25) == 1.25
    assert bench.job_throughput(128, 1, 2.0) == pytest.approx(64000.0)


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                          text=True, timeout=300, env=env, cwd=ROOT)


def test_reference_arm_prints_its_line():
    r = _run_bench(["--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "1",
                    "--cpu-seconds", "0.5"])
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["higher_is_better"] is True


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "1"],
                   {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_ffn_roofline_arithmetic():
    """The FFN's two roofs: bytes at the copy rate and FLOPs at the tensor
    rate of its operand type (twice bf16 for 8-bit and 4-bit weights), the
    higher roof naming the bound, and the same achieved rate against the
    power-capped (sustained) figure."""
    import numpy as np
    from combine_softmax_top_b200 import workloads as W
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1200.0}
    spec = W.spec("prefill")
    counts = np.full(spec.E, spec.T * spec.k // spec.E, dtype=np.int64)
    flops = bench.ffn_flops(spec, int(counts.sum()))
    assert flops == 6.0 * spec.H * spec.I * spec.T * spec.k
    ms = 3.0
    r = bench.ffn_roofline(spec, counts, ms, peaks, "measured")
    t = r["tensor"]
    assert t["peak"] == 3000.0 and t["peak_sustained"] == 2400.0
    assert t["achieved"] == pytest.approx(flops / 3e-3 / 1e12)
    assert t["frac"] == pytest.approx(t["achieved"] / 3000.0)
    assert t["frac_sustained"] == pytest.approx(t["achieved"] / 2400.0)
    abytes, touched = bench.ffn_algorithmic_bytes(spec, counts)
    assert touched == spec.E and r["hbm"]["achieved"] == pytest.approx(abytes / 3e-3 / 1e9)
    # 256 rows per expert: 5.77 TFLOP against 13 GB (weights, rows, h twice,
    # y): 1.92 ms at 3 PFLOP/s, 2.16 ms at 6 TB/s, so the byte roof is higher
    t_tc, t_hbm = flops / 3000e12, abytes / 6000e9
    assert t_hbm > t_tc and r["bound"] == "hbm"
    assert bench.ffn_roofline(spec, counts, ms, dict(peaks, hbm_gbs=8000.0), "measured")["bound"] == "tensor"
    dec = W.spec("decode")
    dcounts = np.zeros(dec.E, dtype=np.int64)
    dcounts[: dec.T * dec.k // 4] = 4
    rd = bench.ffn_roofline(dec, dcounts, 1.7, peaks, "measured")
    assert rd["bound"] == "hbm"                       # 4 rows per expert: weight streaming
    assert rd["tensor"]["peak"] == 3000.0             # e4m3 weights: twice bf16
    bf = W.spec("skew")
    rb = bench.ffn_roofline(bf, np.full(bf.E, bf.T * bf.k // bf.E), 1.0, peaks, "measured")
    assert rb["tensor"]["peak"] == 1500.0 and rb["tensor"]["peak_sustained"] == 1200.0


def test_ncu_dram_bytes_per_launch(tmp_path):
    """DRAM bytes per launch from an ncu --csv metrics log: read + write per
    launch ID, units scaled, other kernels and metrics ignored, the banner
    lines before the header skipped."""
    cols = ["ID", "Process ID", "Process Name", "Host Name", "Kernel Name", "Context", "Stream",
            "Block Size", "Grid Size", "Device", "CC", "Section Name", "Metric Name", "Metric Unit",
            "Metric Value"]

    def row(i, kern, metric, unit, value):
        return [str(i), "1", "python3", "host", kern, "1", "7", "(352, 1, 1)", "(148, 1, 1)", "0", "10.0",
                "Command line profiler metrics", metric, unit, value]

    rows = [row(0, "void ffn_tc_kernel<1, 16>(TcParams)", "dram__bytes_read.sum", "Gbyte", "1.5"),
            row(0, "void ffn_tc_kernel<1, 16>(TcParams)", "dram__bytes_write.sum", "Mbyte", "100"),
            row(0, "void ffn_tc_kernel<1, 16>(TcParams)", "gpu__time_duration.sum", "us", "900"),
            row(1, "void combine_kernel<1, 1>(Args)", "dram__bytes_read.sum", "Gbyte", "9"),
            row(2, "void ffn_tc_kernel<1, 16>(TcParams)", "dram__bytes_read.sum", "byte", "1,300,000,000"),
            row(2, "void ffn_tc_kernel<1, 16>(TcParams)", "dram__bytes_write.sum", "Kbyte", "100000")]
    p = tmp_path / "launches.csv"
    with open(p, "w") as f:
        f.write("==PROF== Connected to process 1\n")
        for r in [cols] + rows:
            f.write(",".join(f'"{c}"' for c in r) + "\n")
    mean, n = bench.ncu_dram_bytes(str(p), "ffn_tc_kernel")
    assert n == 2
    assert mean == pytest.approx((1.5e9 + 100e6 + 1.3e9 + 100e6) / 2)
    with pytest.raises(ValueError):
        bench.ncu_dram_bytes(str(p), "ffn_pair")


def test_recorded_traffic_only_for_the_current_source(tmp_path, monkeypatch):
    """A recorded DRAM/algorithmic ratio is applied to a launch's algorithmic
    bytes only while the FFN sources hash as they did at capture."""
    rec = {"grouped_ffn/decode": {"source_sha": "abc", "traffic_ratio": 1.01}}
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(p))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "abc")
    assert bench.recorded_traffic("grouped_ffn/decode", 1_000_000) == 1_010_000
    assert bench.recorded_traffic("grouped_ffn/prefill", 1_000_000) is None
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "changed")
    assert bench.recorded_traffic("grouped_ffn/decode", 1_000_000) is None
