"""EpGroup's exchange on the CPU: 2 and 3 gloo ranks as processes, the kernels
replaced by oracle-based stand-ins (so no GPU is needed), one rank with an empty
batch.  Checks the rows each rank receives, the per-(source, expert) counts and the
combine results against the oracle, for FP8 and BF16 payloads, for both transports:
the all-to-all one, and the peer one (receive buffers in POSIX shared memory stand
for IPC-mapped GPU memory; the stand-in kernels store and load through the pointer
tables)."""
import multiprocessing as mp
import socket

import pytest


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("transport", ["nccl", "peer"])
@pytest.mark.parametrize("world", [2, 3])
def test_ep_group_exchange_on_cpu(tmp_path, world, transport):
    import ep_cpu_worker

    target = ep_cpu_worker.run if transport == "nccl" else ep_cpu_worker.run_peer
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():  # only our own children
            p.kill()
            p.join()
    results = [(tmp_path / f"rank{r}.txt").read_text() if (tmp_path / f"rank{r}.txt").exists()
               else "missing" for r in range(world)]
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    assert results == ["ok"] * world, results
