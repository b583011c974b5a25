"""Host side of the column-parallel layer (ColumnParallelLinear) over two gloo
ranks on the CPU: shard offsets and the full width from the ranks' shard
widths, the exchange of buffer handles (each rank maps every other rank's
buffer and never its own), the pointers handed to the kernel call (every
rank's output buffer, alternating between two per call, and every rank's
flag array), the alternation of output buffers, and the collective
teardown order.  The
shared-memory calls and the kernel call are replaced by recording fakes."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class FakeIpc:
    """Buffers are fake addresses; a handle names its owner's address."""

    def __init__(self, rank):
        self.rank = rank
        self.log = []

    def malloc(self, nbytes):
        ptr = (self.rank + 1) << 32
        self.log.append(("malloc", nbytes))
        return ptr, f"buffer-of-rank-{self.rank}".encode().ljust(64, b"\0")

    def open(self, handle):
        owner = int(handle.rstrip(b"\0").decode().rsplit("-", 1)[1])
        self.log.append(("open", owner))
        return ((owner + 1) << 32) + (1 << 20)  # another process maps it at another address

    def close(self, ptr):
        self.log.append(("close", ptr))

    def free(self, ptr):
        self.log.append(("free", ptr))


def _rank_main(rank, world, port, widths, q):
    import datetime

    import torch.distributed as dist

    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import quantized_gemm_decode_b200 as qgd
        from quantized_gemm_decode_b200 import linear

        calls = []
        qgd.qlinear_tp_bf16 = lambda *a, **kw: calls.append((a, kw))  # the kernel call, recorded
        N, K = widths[rank], 512
        weights = (torch.zeros((N, K), dtype=torch.uint8), torch.ones(N), None)
        ipc = FakeIpc(rank)
        layer = linear.ColumnParallelLinear(None, "fp8_dynamic", max_m=8, weights=weights, ipc=ipc)
        x = torch.zeros((4, K), dtype=torch.bfloat16)
        bufs = [layer.launch(x) for _ in range(3)] + [layer.launch(torch.zeros((0, K), dtype=torch.bfloat16))]
        layer.close()
        q.put((rank, layer.col0, layer.ldy, layer.own, list(ipc.log), bufs, layer.calls,
               [(kw["rank"], kw["ranks"], kw["col0"], kw["ldy"], kw["ys"], kw["flags"])
                for _, kw in calls], layer.out_bytes, layer.flags_off, None))
    except Exception as exc:
        q.put((rank,) + (None,) * 10 + (repr(exc),))
    finally:
        dist.destroy_process_group()


def test_column_parallel_plumbing_over_gloo():
    world, widths = 2, [384, 256]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, widths, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=180) for _ in procs], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, col0, ldy, own, log, bufs, ncalls, calls, out_bytes, flags_off, exc in res:
        assert exc is None, f"rank {r}: {exc}"
        assert col0 == sum(widths[:r]) and ldy == sum(widths)
        assert own == (r + 1) << 32
        peer = 1 - r
        peer_ptr = ((peer + 1) << 32) + (1 << 20)
        # one buffer of two outputs [8, 640] bf16 and the flags (2 entries + the counter), each 256-byte aligned
        assert out_bytes == 8 * 640 * 2 and flags_off == 2 * 10240
        assert log[0] == ("malloc", flags_off + 256)
        assert log[1:] == [("open", peer), ("close", peer_ptr), ("free", own)]
        assert bufs == [0, 1, 0, 1] and ncalls == 4         # the empty call takes a buffer turn, launches nothing
        assert len(calls) == 3
        base = {r: own, peer: peer_ptr}
        for i, (rank, ranks, c0, ld, ys, flags) in enumerate(calls):
            assert (rank, ranks, c0, ld) == (r, 2, col0, ldy)
            off = (i & 1) * 10240
            assert ys == [base[0] + off, base[1] + off]
            assert flags == [base[0] + flags_off, base[1] + flags_off]


def test_single_process_needs_no_group():
    from quantized_gemm_decode_b200 import linear

    ipc = FakeIpc(0)
    layer = linear.ColumnParallelLinear(None, "block_fp8", max_m=4,
                                        weights=(torch.zeros((256, 512), dtype=torch.uint8), torch.ones(2, 4), None),
                                        ipc=ipc)
    assert (layer.G, layer.rank, layer.col0, layer.ldy) == (1, 0, 0, 256)
    assert layer.bases == [layer.own]
    layer.close()
    assert [e[0] for e in ipc.log] == ["malloc", "free"]
    with pytest.raises(ValueError):
        linear.ColumnParallelLinear(None, "int4", weights=(torch.zeros((16, 16)), None, None), ipc=ipc)
