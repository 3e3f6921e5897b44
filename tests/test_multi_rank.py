"""The N > 1 host path of bench.py on CPU ranks (gloo, world size 2): the real replica driver
(run_replica) with the CUDA parts of a replica replaced by a stand-in that reports fixed
device times, the max over ranks of every timing, the reference arm on rank 0 only, and the
self-launch of `bench.py --gpus N` as N torchrun ranks."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _StubReplica:
    """The interface of bench.Replica with fixed per-rank device times and no GPU: rank r's
    steps take (1 + r) ms, its kernel launches (100 + 10 r) us."""

    def __init__(self, w, dev):
        import torch
        from grouped_query_attention_decode_b200 import inputs
        self.w = w
        self.x = {"lengths": torch.full((w.B,), w.length or 1, dtype=torch.int32)}
        self.lengths = self.x["lengths"].tolist()
        self.ideal = inputs.ideal_kv_bytes(w, self.lengths)
        self.n_copies = 2
        self.rank = int(os.environ["RANK"])
        self.kernel = "split_tc_kernel"
        self.dtype_name = "bf16"
        self.checked = False

    def l2_label(self):
        return "stub"

    def launches_per_step(self):
        return 2

    def check(self):
        self.checked = True

    def time_kernel(self, n, secs):
        return [100.0 + 10 * self.rank] * 5

    def time_steps(self, K, W, barrier=None):
        if barrier is not None:
            barrier()
        return K * (1.0 + self.rank)

    def time_e2e(self, K, W):
        return {"ms_per_step": 2.0 + self.rank, "serial_ms_per_step": 2.5, "api_only_ms_per_step": 1.5,
                "copies_only_ms_per_step": 0.1, "h2d": 10, "d2h": 20}

    def read_stream(self):
        return {"gbs": 7000.0, "how": "stub"}


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK="0")
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    got = bench.max_over_ranks(1.5 + rank, dist, "cpu")
    args = bench.parse(["--gpus", "2", "--steps", "4", "--warmup", "3", "--also",
                        "t5xxl_g8", "--no-cpu-baseline", "--no-clocks"])
    res = bench.run_replica(args, rank, world, 0, "cpu", dist, _StubReplica)
    dist.barrier()
    dist.destroy_process_group()

    class A:
        workload = "tiny_fp32"
        steps = 1
        warmup = 3
    ref = bench.bench_reference(A, rank, world)
    q.put((rank, got, ref is None, res))


@pytest.mark.timeout(300)
def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=240) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]
    assert res[0][2] is False and res[1][2] is True   # rank 0 reports, rank 1 does no work
    line, other = res[0][3], res[1][3]
    assert other is None
    ideal = 2 * 16 * 4096 * 8 * 128 * 2
    # the slowest rank (2 ms per step) sets the whole job's time; value counts both replicas
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["ms_per_step"] == pytest.approx(2.0)
    assert line["value"] == pytest.approx(2 * ideal / 2e-3 / 1e9, rel=1e-4)
    assert line["gpu_launches"] == 2 * 4
    assert line["e2e"]["ms_per_step"] == pytest.approx(3.0)
    assert line["roofline"]["avg_launch_us_max_over_ranks"] == pytest.approx(110.0)
    assert line["also"]["workload"] == "t5xxl_g8"
    assert line["also"]["us_per_step"] == pytest.approx(2000.0)


def test_gpus_n_relaunches_as_n_ranks():
    sys.path.insert(0, ROOT)
    import bench
    cmd = bench.launcher_argv(4, ["--gpus", "4", "--steps", "20"], port=12345)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd and "--master-port=12345" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "20"] and cmd[-5].endswith("bench.py")
