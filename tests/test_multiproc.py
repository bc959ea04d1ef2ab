"""The N > 1 benchmark path on CPU: two gloo ranks, each timing its own replica; the job time is
the max over ranks and the job value counts every rank's work (weak scaling)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        mine = [10.0 + rank, 1.0 * (world - rank), 3.0]
        q.put((rank, bench.reduce_max(mine, torch.device("cpu"))))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [11.0, 2.0, 3.0]


def test_whole_job_value_is_weak_scaling():
    import bench
    one = bench.whole_job_tflops(10 ** 12, 100, 1, 1000.0)
    assert one == pytest.approx(100.0)
    # two ranks, slower one at 1.25 s: twice the work over the max time
    assert bench.whole_job_tflops(10 ** 12, 100, 2, 1250.0) == pytest.approx(160.0)


def test_single_process_reduce_is_identity():
    import torch
    import bench
    assert bench.reduce_max([1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]


def test_packed_step_buffers_hold_every_tensor_aligned_and_apart():
    # the end-to-end step moves a step's inputs (outputs) as one buffer: every tensor must be a
    # view at a 256-byte aligned offset, of its own shape and type, and no two views may overlap
    import torch
    import bench
    like = {"q": torch.zeros(2, 8, 33, 40, dtype=torch.bfloat16), "x": torch.zeros(2, 5, 3, 3),
            "g": torch.zeros(7), "lat": torch.zeros(1, 4, 8, 8)}
    blob, views = bench._packed(like, list(like))
    spans = []
    for k, t in like.items():
        v = views[k]
        assert v.shape == t.shape and v.dtype == t.dtype and v.is_contiguous()
        off = v.data_ptr() - blob.data_ptr()
        assert off % 256 == 0
        spans.append((off, off + v.numel() * v.element_size()))
        v.fill_(1)
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= blob.numel()
    assert float(views["q"].float().sum()) == like["q"].numel()
