"""The N > 1 bench path on CPU: two gloo ranks (replicas) agree on the max
elapsed time and the summed units, and only rank 0 prints.  CPU only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist = bench.init_dist("gloo")
    elapsed, units = bench.aggregate(dist, 10.0 + 5.0 * rank, 256.0)
    bench.barrier(dist)
    dist.destroy_process_group()
    q.put((rank, elapsed, units))


def test_two_rank_replica_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, elapsed, units in res:
        assert elapsed == 15.0          # max over ranks
        assert units == 512.0           # sum over the two replicas


def test_single_process_aggregation_is_identity():
    import bench
    assert bench.aggregate(None, 3.5, 7.0) == (3.5, 7.0)


def test_oracle_extrapolation_arithmetic():
    import bench
    W = bench.workload("full_b1")
    tps, step_s, block_s = bench.oracle_tokens_per_s(W, layer_s=2.0, head_row_s=0.1, steps_per_block=10)
    assert step_s == pytest.approx(30 * 2.0 + 256 * 0.1)
    assert block_s == pytest.approx(10 * step_s + 30 * 2.0)
    assert tps == pytest.approx(256 / block_s)


REFERENCE_KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                  "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _run_reference(cmd, env_extra=None, timeout=600):
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **(env_extra or {}))
    return subprocess.run([sys.executable] + cmd, cwd=root, env=env, capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` times the oracle on the host cores (no GPU needed) and prints one JSON line
    with the contract's keys; its cpu_baseline and e2e describe the same run."""
    import json
    r = _run_reference(["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert REFERENCE_KEYS <= set(d)
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 0
    assert d["value"] > 0 and d["higher_is_better"] is True and d["config"]["workload"] == "full_b1"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_under_torchrun_prints_on_rank_0_only():
    port = _free_port()
    r = _run_reference(["-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
                        "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1 and '"impl": "reference"' in lines[0]


def test_clock_sampler_keeps_samples_of_a_short_region(tmp_path, monkeypatch):
    """The bench's clock record: with a fake nvidia-smi writing a sample every
    20 ms, a timed region shorter than the interval still gets one sample
    (the first after its end), and samples before the region are dropped."""
    import stat
    import time

    import bench
    fake = tmp_path / "nvidia-smi"
    fake.write_text(
        "#!" + sys.executable + "\n"
        "import sys, time\n"
        "path = sys.argv[sys.argv.index('-f') + 1]\n"
        "i = 0\n"
        "while True:\n"
        "    with open(path, 'a') as fh:\n"
        "        mhz = 1000 if i == 0 else 1965\n"
        "        fh.write(f'0, {mhz}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Active\\n')\n"
        "    i += 1\n"
        "    time.sleep(0.02)\n")
    fake.chmod(fake.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])
    clk = bench.ClockSampler(0)
    clk.__enter__()
    time.sleep(0.05)          # samples before the region: dropped
    clk.mark()
    clk.stop()                # a region shorter than the interval
    clk.__exit__(None, None, None)
    s = clk.summary()
    assert s["samples"] >= 1
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_kernel_rooflines_name_the_kernels_in_use():
    """The per-class rooflines name the kernel the library runs for the pass
    size: CTA pairs for attention (16/8 heads), the canvas-size dense split-K
    and gate/up; the batch-16 passes run both expert projections on pairs."""
    import bench
    from discrete_text_diffusion_b200 import synth
    model = synth.WORKLOADS["full_b16"]["model"]
    peaks = {"hbm_gbs": 6544.0, "bf16_tflops": 1653.0, "bf16_tflops_sustained": 1396.4}
    bd = {c: (240, 10.0) for c in ["attention", "moe_up", "moe_down", "dense_gemm", "lm_head", "sampler_rows"]}
    b1 = bench.kernel_rooflines(model, 1, 256, [(8192, 7)], 14.8, bd, peaks, "measured")
    b16 = bench.kernel_rooflines(model, 16, 256, [(4096, 12)], 61.5, bd, peaks, "measured")
    assert b1["attention"]["kernel"].startswith("attn_tc2_kernel")
    assert b1["dense_gemm"]["kernel"].startswith("gemm_tc2_kernel")
    assert b1["moe_up"]["kernel"].startswith("gemm_tc2_grouped_kernel")
    assert b1["moe_down"]["kernel"].startswith("gemm_tc_kernel")
    assert b16["moe_up"]["kernel"].startswith("gemm_tc2_grouped_kernel")
    assert b16["moe_down"]["kernel"].startswith("gemm_tc2_grouped_kernel")
    assert b16["dense_gemm"]["kernel"].startswith("gemm_tc_kernel")
    for r in list(b1.values()) + list(b16.values()):
        assert 0 < r["frac"] and r["launches"] == 240
