"""The N-GPU benchmark path runs independent replicas (the layer has no
exchange step); the only collective is the max-over-ranks of the timings.
Checked here with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (r + 1) ms, 10 * (r + 1) ms and 3 ms on its three timers
        got = bench.max_over_ranks([rank + 1.0, 10.0 * (rank + 1), 3.0], world, torch.device("cpu"))
        q.put((rank, got, bench.job_throughput(2e12, world, got[0])))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, thr in res:
        assert got == [2.0, 20.0, 3.0]                 # the slowest replica's times, on every rank
        assert thr == pytest.approx(2e12 * 2 / 2e-3 / 1e12)


def test_single_rank_is_identity():
    assert bench.max_over_ranks([1.5, 2.5], 1, torch.device("cpu")) == [1.5, 2.5]
    assert bench.job_throughput(1e12, 1, 1.0) == pytest.approx(1000.0)


class _StubLib:
    """Stands in for the CUDA library: size helpers are real, every launch
    entry point returns OK without doing anything."""

    def __init__(self, real):
        self.real = real

    def __getattr__(self, name):
        if name in ("nvfp4_sf_bytes", "nvfp4_codes_bytes", "w4a4_gemm_workspace_bytes",
                    "nvfp4_gemm_workspace_bytes", "nvfp4_launch_count", "nvfp4_status_string"):
            return getattr(self.real, name)
        return lambda *a, **k: 0


def _flow_main(rank: int, world: int, port: int, q):
    """The whole N-rank benchmark flow with the CUDA pieces stubbed: rank r's
    events report r + 1 ms, so the job time must be the slowest rank's."""
    import types
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from nvfp4_w4a4_quantized_06_b200 import native
        native._lib = _StubLib(native.lib())
        native._require_cuda = lambda *ts: None
        native._stream = lambda: 0
        native.last_device_status = lambda: 0

        class Ev:
            def __init__(self, *a, **k):
                pass

            def record(self, *a, **k):
                pass

            def elapsed_time(self, other):
                return float(rank + 1)

        class Stream:
            cuda_stream = 0

            def __init__(self, *a, **k):
                pass

            def wait_stream(self, other):
                pass

            def wait_event(self, ev):
                pass

        import contextlib
        torch.cuda.Event = Ev
        torch.cuda.Stream = Stream
        torch.cuda.stream = lambda s: contextlib.nullcontext()
        torch.cuda.synchronize = lambda *a, **k: None
        torch.cuda.current_stream = lambda *a, **k: Stream()
        torch.cuda.empty_cache = lambda: None
        torch.Tensor.pin_memory = lambda self, *a, **k: self
        args = types.SimpleNamespace(gpus=world, steps=3, warmup=3, impl="native", workload="decode_out_proj",
                                     headline_only=True, no_cpu_baseline=True, no_e2e=False, oracle_table=False)
        out = bench.run_native(args, rank, world, torch.device("cpu"))
        # the JSON line's contract: every key the benchmark promises is there
        missing = [k for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                               "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                               "roofline", "roofline_quant", "e2e", "gpu_launches", "clocks") if k not in out]
        missing += ["roofline." + k for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")
                    if k not in out["roofline"]]
        missing += ["e2e." + k for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step")
                    if k not in out["e2e"]]
        missing += ["config.workload"] if "workload" not in out["config"] else []
        q.put((rank, out["n_gpus"], out["ms_per_step"], out["value"], out["e2e"]["ms_per_step"],
               out["config"]["parallelism"], missing))
    finally:
        dist.destroy_process_group()


def test_benchmark_flow_on_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_flow_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = bench.W.WORKLOADS["decode_out_proj"]
    for rank, n, ms, value, e2e_ms, par, missing in res:
        assert not missing, missing
        assert n == 2 and par == "replicas x2"
        assert ms == pytest.approx(2.0 / 3, rel=1e-3)         # the slower rank's 2 ms over 3 steps
        assert value == pytest.approx(bench.job_throughput(wl.flops, 2, ms), rel=1e-2)
        assert e2e_ms > 0
