"""The multi-GPU form of the benchmark is replicas only: no collective on the data
path, only the max over ranks of the device time.  This checks that reduction
and the whole-job throughput with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "measured" (10 + r) ms for the step loop and (20 - r) ms end to end
        got = bench.max_over_ranks([10.0 + rank, 20.0 - rank], "cpu", world)
        value = bench.job_throughput(4096, 5, world, got[0])
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in results:
        assert got == [11.0, 20.0]            # every rank sees the slowest rank's times
        assert value == pytest.approx(4096 * 5 * 2 / 0.011)


def test_single_rank_is_identity():
    assert bench.max_over_ranks([1.5, 2.5], "cpu", 1) == [1.5, 2.5]
    assert bench.job_throughput(100, 2, 1, 1000.0) == 200.0


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup, seed, gpus, out_dtype = 1, 0, 0, 2, "bf16"

    from mixture_experts_routing_02_b200 import synthetic as syn
    assert bench.run_reference(A, syn.TINY) == 0      # returns at once, no work, no output


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    """--impl reference on rank 0: the oracle timed on a bounded sample, one JSON line with the
    keys the driver reads (no GPU needed)."""
    import json
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.setenv("WORLD_SIZE", "1")

    class A:
        steps, warmup, seed, gpus, out_dtype = 1, 0, 0, 1, "bf16"

    from mixture_experts_routing_02_b200 import synthetic as syn
    assert bench.run_reference(A, syn.TINY) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["higher_is_better"] is True and d["vs_baseline"] is None and d["steps"] == 1
    assert d["config"]["workload"] == "tiny"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_clock_sampler_with_a_fake_nvml(monkeypatch):
    """The bench's clock sampler, run against a fake NVML on the CPU: it samples on its own thread
    while the timed work runs, reports the median SM clock and the throttle reasons it saw, and
    only reads the GPU's settings (the fake has no setter to call)."""
    import sys
    import time
    import types

    clocks = iter([1965, 1500, 1400, 1500] + [1450] * 10000)
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByPciBusId=lambda bus: "gpu0",
        nvmlDeviceGetMaxClockInfo=lambda h, kind: 1965,
        nvmlDeviceGetClockInfo=lambda h, kind: next(clocks),
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x4,      # sw_power_cap
    )
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    props = types.SimpleNamespace(pci_domain_id=0, pci_bus_id=0x1B, pci_device_id=0)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda dev: props)
    s = bench.ClockSampler(0).__enter__()
    time.sleep(0.1)
    s.__exit__(None, None, None)
    out = s.summary()
    assert out["samples"] >= 5 and out["sm_max_mhz"] == 1965
    assert out["sm_mhz"] == 1450 and out["reasons"] == ["sw_power_cap"]
