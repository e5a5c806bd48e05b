"""EpGroup across processes: two ranks, each its own process on the one visible GPU,
exchanging through gloo (host memory).  The kernels of the two processes never wait
on each other; only the host-side collectives couple them.  Every rank checks its
received rows and its combine result bit for bit against the oracle."""
import multiprocessing as mp
import os
import socket

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [1, 2])
def test_ep_group_dispatch_combine(tmp_path, world):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import ep_worker

    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=ep_worker.run, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():  # only our own children
            p.kill()
            p.join()
    results = [(tmp_path / f"rank{r}.txt").read_text() if (tmp_path / f"rank{r}.txt").exists()
               else "missing" for r in range(world)]
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    assert results == ["ok"] * world, results


def test_ep_group_peer_transport_one_rank(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import ep_worker

    ctx = mp.get_context("spawn")
    p = ctx.Process(target=ep_worker.run_peer, args=(0, 1, _free_port(), str(tmp_path)))
    p.start()
    p.join(timeout=240)
    if p.is_alive():  # only our own child
        p.kill()
        p.join()
    assert p.exitcode == 0
    assert (tmp_path / "rank0.txt").read_text() == "ok"


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs two or more GPUs (one process per GPU)")
def test_ep_group_peer_transport_across_gpus(tmp_path):
    import ep_worker

    world = min(torch.cuda.device_count(), 4)
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=ep_worker.run_peer_multi, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    for p in procs:
        if p.is_alive():  # only our own children
            p.kill()
            p.join()
    results = [(tmp_path / f"rank{r}.txt").read_text() if (tmp_path / f"rank{r}.txt").exists()
               else "missing" for r in range(world)]
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    assert results == ["ok"] * world, results
