"""Column-parallel layer calls with the all-gather fused into the Swap-AB
epilogue (qlinear_tp_bf16 + qgd_tp_wait), checked against the oracle of the
unsharded layer.

The library's own extension of the pages' single-GPU operation: the weight
rows (output columns) are split over G ranks, each rank's kernel stores its
columns into every rank's full output and then advances its call count
and writes it into every rank's flag array.  With one GPU the ranks are emulated in one process: all G
calls run first, one after another, each writing all G outputs and flag
arrays; only then are the G waits enqueued, so no kernel ever waits for a
kernel that has not yet finished.  The IPC test runs two processes on the
same GPU in the same order (a host barrier between the calls and the waits).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import quantized_gemm_decode_b200 as qgd
from quantized_gemm_decode_b200 import synth
from quantized_gemm_decode_b200.linear import ColumnParallelLinear, quantize_weight
from paritylib import bf16_to_f64, check_fp8_tolerance, check_within_one_ulp

pytestmark = pytest.mark.gpu

FMTS = {"fp8_dynamic": qgd.FMT_FP8_DYNAMIC, "w8a8_int8": qgd.FMT_W8A8_INT8, "block_fp8": qgd.FMT_BLOCK_FP8,
        "mxfp8": qgd.FMT_MXFP8, "nvfp4": qgd.FMT_NVFP4}
SENTINEL = -1  # 0xFFFF: a bf16 NaN; any element the kernels do not write stays NaN


@pytest.fixture(autouse=True)
def _clean():
    qgd.lib()
    for f in FMTS.values():
        qgd.qgd_set_override(f)
        qgd.qgd_set_fused_override(f, -1)
    qgd.qgd_clear_device_error()
    yield
    for f in FMTS.values():
        qgd.qgd_set_override(f)
        qgd.qgd_set_fused_override(f, -1)


def oracle_layer(fmt: str, x: torch.Tensor, w: torch.Tensor):
    """The unsharded layer: the oracle's quantization of x and W, then its product."""
    if fmt == "block_fp8":
        xq, sx = oracle.quant_groups(x, 128)
        wq, sw = oracle.quant_blocks(w, 128)
        return oracle.gemm_blockscaled(xq, sx, wq, sw, 128)
    if fmt == "mxfp8":
        xq, sx = oracle.quant_mx(x)
        wq, sw = oracle.quant_mx(w)
        return oracle.gemm_mx(xq, sx, wq, sw)
    if fmt == "nvfp4":
        return oracle.gemm_nv(*oracle.quant_nv(x), *oracle.quant_nv(w))
    qt = oracle.INT8 if fmt == "w8a8_int8" else oracle.E4M3
    xq, sx = oracle.quant_rows(x, qt)
    wq, sw = oracle.quant_rows(w, qt)
    return oracle.gemm_rowscaled(xq, sx, wq, sw, qt)


def check_layer(fmt: str, y: torch.Tensor, yref: np.ndarray, bound: np.ndarray, K: int, what: str) -> None:
    yy = bf16_to_f64(y)
    if fmt == "w8a8_int8":
        check_within_one_ulp(yy, yref, what)
    else:
        check_fp8_tolerance(yy, yref, bound, K, what)


def run_emulated(fmt: str, Ms, widths, K: int, seed: int, max_m: int = None):
    """G = len(widths) ranks on one GPU, one call per entry of Ms (outputs
    alternate between two buffers).  Every rank's full output is checked
    against the oracle after every call, and its flags against the count."""
    F = FMTS[fmt]
    G, ldy = len(widths), sum(widths)
    col0 = [sum(widths[:r]) for r in range(G)]
    max_m = max_m or max(Ms)
    w = synth.weights(ldy, K, seed)
    shards = [quantize_weight(w[c:c + n].cuda(), fmt) for c, n in zip(col0, widths)]
    outs = [[torch.full((max_m, ldy), SENTINEL, dtype=torch.int16, device="cuda") for _ in range(G)]
            for _ in range(2)]
    flags = [torch.zeros(G + 1, dtype=torch.int32, device="cuda") for _ in range(G)]  # + the call counter
    wss = [qgd.Workspace(qgd.qgd_tp_workspace_size(F, max_m, n, K)) for n in widths]
    for call, M in enumerate(Ms):
        count, buf = call + 1, call & 1
        for o in outs[buf]:
            o.fill_(SENTINEL)
        x = synth.activations(M, K, seed + 7 * call, outliers=True)
        xd = x.cuda()
        for r in range(G):
            wq, sw, sb = shards[r]
            qgd.qlinear_tp_bf16(F, xd, wq, sw, sb, ranks=G, rank=r, col0=col0[r], ldy=ldy, ys=outs[buf],
                                flags=flags, ws=wss[r])
        for r in range(G):
            qgd.qgd_tp_wait(flags[r], G)
        torch.cuda.synchronize()
        assert qgd.qgd_device_error() == 0
        for r in range(G):
            assert flags[r].cpu().tolist() == [count] * (G + 1), f"rank {r} flags after call {call}"
            # the completion counter (last word of the 64 KiB header) is back to zero
            assert int(wss[r].buf[65536 - 4:65536].view(torch.int32).item()) == 0
        yref, bound = oracle_layer(fmt, x, w)
        for r in range(G):
            full = outs[buf][r]
            check_layer(fmt, full[:M].view(torch.bfloat16), yref, bound, K,
                        f"{fmt} rank {r}/{G} call {call} M={M} widths={widths}")
            assert bool((full[M:] == SENTINEL).all()), "rows past M were written"


CASES = [
    ("fp8_dynamic", [1, 7], [256, 384], 1024),
    ("fp8_dynamic", [32, 16, 3], [512, 128, 256, 640], 2048),
    ("w8a8_int8", [5, 32], [384, 256, 512], 1024),
    ("block_fp8", [1, 24], [256, 512], 1024),
    ("block_fp8", [8], [128, 128, 256, 128, 384, 128, 256, 128], 512),
    ("mxfp8", [4, 33], [256, 512], 1024),
    ("nvfp4", [2, 64], [512, 256, 256], 2048),
    ("nvfp4", [100, 128], [256, 384], 1024),
    ("mxfp8", [128, 65], [384, 256, 128], 1024),
    ("fp8_dynamic", [100], [256, 256], 1024),
]


@pytest.mark.parametrize("fmt,Ms,widths,K", CASES,
                         ids=[f"{c[0]}-G{len(c[2])}-M{'_'.join(map(str, c[1]))}" for c in CASES])
def test_tp_emulated_ranks_match_oracle(fmt, Ms, widths, K):
    run_emulated(fmt, Ms, widths, K, seed=len(widths) * 100 + K)


SW, GRID, PERS = qgd.VARIANT_SWAP_AB, qgd.SCHEDULE_GRID, qgd.SCHEDULE_PERSISTENT
TP_PLANS = [
    (SW, 1, qgd.REDUCE_LAST_CTA, 0, 0, GRID, 1, 1),
    (SW, 4, qgd.REDUCE_LAST_CTA, 0, 0, GRID, 1, 2),
    (SW, 8, qgd.REDUCE_ATOMIC, 0, 0, GRID, 1, 1),
    (SW, 3, qgd.REDUCE_CLUSTER, 0, 0, GRID, 1, 1),
    (SW, 4, qgd.REDUCE_TWO_PASS, 0, 0, GRID, 1, 1),         # taken as last-arriving CTA
    (SW, 1, qgd.REDUCE_LAST_CTA, 0, 0, PERS, 2, 2),
    (qgd.VARIANT_STANDARD, 1, qgd.REDUCE_LAST_CTA, 0, 256, PERS, 1, 1),  # taken as Swap-AB
]


@pytest.mark.parametrize("fused", [0, 1])
@pytest.mark.parametrize("plan", TP_PLANS, ids=[f"v{p[0]}-s{p[1]}-r{p[2]}-sch{p[5]}-k{p[7]}" for p in TP_PLANS])
def test_tp_plans(plan, fused):
    for fmt in ("fp8_dynamic", "block_fp8"):
        qgd.qgd_set_override(FMTS[fmt], *plan)
        qgd.qgd_set_fused_override(FMTS[fmt], fused)
    run_emulated("fp8_dynamic", [9], [384, 256], 2048, seed=11)
    run_emulated("block_fp8", [17], [256, 384], 1024, seed=12)


def test_tp_single_rank_is_the_plain_layer_call():
    # one rank: the full output is this rank's own, bit-identical to qlinear_bf16 with the same plan
    F, M, N, K = qgd.FMT_FP8_DYNAMIC, 12, 768, 2048
    qgd.qgd_set_override(F, SW, 2, qgd.REDUCE_LAST_CTA, 0, 0, GRID, 1, 1)
    x = synth.activations(M, K, 5).cuda()
    wq, sw, _ = quantize_weight(synth.weights(N, K, 5).cuda(), "fp8_dynamic")
    y = torch.full((M, N + 64), SENTINEL, dtype=torch.int16, device="cuda")
    flags = torch.tensor([2, 2], dtype=torch.int32, device="cuda")  # two calls already made
    ws = qgd.Workspace(qgd.qgd_tp_workspace_size(F, M, N, K))
    qgd.qlinear_tp_bf16(F, x, wq, sw, None, ranks=1, rank=0, col0=64, ldy=N + 64, ys=[y], flags=[flags], ws=ws)
    qgd.qgd_tp_wait(flags, 1)
    y_plain = qgd.qlinear_bf16(F, x, wq, sw)
    torch.cuda.synchronize()
    assert qgd.qgd_device_error() == 0 and flags.tolist() == [3, 3]
    assert torch.equal(y[:, 64:], y_plain.view(torch.int16))
    assert bool((y[:, :64] == SENTINEL).all())


def test_tp_wait_gives_up_on_a_flag_nobody_sets():
    # bounded wait: about one second, then device error 6 and the kernel returns
    flags = torch.tensor([0, 1], dtype=torch.int32, device="cuda")  # count 1, nobody has reached it
    qgd.qgd_tp_wait(flags, 1)
    torch.cuda.synchronize()
    assert qgd.qgd_device_error() == 6
    qgd.qgd_clear_device_error()
    # the context is still usable: a count past this rank's own also ends the wait
    flags.copy_(torch.tensor([5, 4], dtype=torch.int32))
    qgd.qgd_tp_wait(flags, 1)
    torch.cuda.synchronize()
    assert qgd.qgd_device_error() == 0


def test_tp_graph_replay_advances_the_count():
    # the count lives on the device: a captured pair of ranks replays correctly
    F, M, K, widths = qgd.FMT_FP8_DYNAMIC, 4, 1024, [256, 384]
    G, ldy = 2, sum(widths)
    w = synth.weights(ldy, K, 31)
    shards = [quantize_weight(w[c:c + n].cuda(), "fp8_dynamic") for c, n in ((0, 256), (256, 384))]
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    outs = [torch.zeros((M, ldy), dtype=torch.int16, device="cuda") for _ in range(G)]
    flags = [torch.zeros(G + 1, dtype=torch.int32, device="cuda") for _ in range(G)]
    wss = [qgd.Workspace(qgd.qgd_tp_workspace_size(F, M, n, K)) for n in widths]

    def step():
        for r in range(G):
            qgd.qlinear_tp_bf16(F, x, *shards[r], ranks=G, rank=r, col0=sum(widths[:r]), ldy=ldy, ys=outs,
                                flags=flags, ws=wss[r])
        for r in range(G):
            qgd.qgd_tp_wait(flags[r], G)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # count 1
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()  # captured, not run
    for rep in range(3):
        xr = synth.activations(M, K, 40 + rep)
        x.copy_(xr.cuda())
        g.replay()
        torch.cuda.synchronize()
        assert qgd.qgd_device_error() == 0
        for r in range(G):
            assert flags[r].cpu().tolist() == [rep + 2] * (G + 1)
        yref, bound = oracle_layer("fp8_dynamic", xr, w)
        for r in range(G):
            check_layer("fp8_dynamic", outs[r].view(torch.bfloat16), yref, bound, K, f"replay {rep} rank {r}")


def test_tp_rejects_bad_descriptors():
    F, M, N, K = qgd.FMT_FP8_DYNAMIC, 4, 256, 512
    x = synth.activations(M, K, 1).cuda()
    wq, sw, _ = quantize_weight(synth.weights(N, K, 1).cuda(), "fp8_dynamic")
    y = torch.zeros((M, 512), dtype=torch.int16, device="cuda")
    flags = torch.zeros(3, dtype=torch.int32, device="cuda")
    ws = qgd.Workspace(qgd.qgd_tp_workspace_size(F, M, N, K))
    common = dict(ranks=2, ys=[y, y], flags=[flags, flags], ws=ws)
    bad = [dict(rank=2, col0=0, ldy=512),       # rank out of range
           dict(rank=0, col0=300, ldy=512),     # shard past the full output
           dict(rank=0, col0=0, ldy=500)]       # ldy not a multiple of 8
    for kw in bad:
        with pytest.raises(qgd.QGDError) as e:
            qgd.qlinear_tp_bf16(F, x, wq, sw, None, **common, **kw)
        assert e.value.status == -1
    xb = synth.activations(40, 1024, 2).cuda()
    wb, swb, _ = quantize_weight(synth.weights(256, 1024, 2).cuda(), "block_fp8")
    with pytest.raises(qgd.QGDError) as e:  # Block_FP8 Swap-AB covers 32 tokens
        qgd.qlinear_tp_bf16(qgd.FMT_BLOCK_FP8, xb, wb, swb, None, rank=0, col0=0, ldy=512,
                            **dict(common, ws=qgd.Workspace(1 << 20)))
    assert e.value.status == -2
    torch.cuda.synchronize()
    assert flags.sum().item() == 0 and qgd.qgd_device_error() == 0


# ---------------------------------------------------------------------------
# Two processes on one GPU through CUDA IPC (the ColumnParallelLinear class)
# ---------------------------------------------------------------------------
def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_rank(rank, world, port, fmt, widths, K, Ms, seed, q):
    import datetime

    import torch.distributed as dist

    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        col0 = sum(widths[:rank])
        w = synth.weights(sum(widths), K, seed)
        layer = ColumnParallelLinear(w[col0:col0 + widths[rank]].cuda(), fmt, max_m=max(Ms))
        outs = []
        for call, M in enumerate(Ms):
            x = synth.activations(M, K, seed + 7 * call).cuda()
            buf = layer.launch(x)
            torch.cuda.synchronize()
            dist.barrier()          # every rank's call has finished before any wait starts
            y = layer.wait(M, buf)
            torch.cuda.synchronize()
            outs.append(y.view(torch.int16).cpu().clone())
            dist.barrier()          # nobody starts the call after next while another still reads
        err = qgd.qgd_device_error()
        layer.close()
        q.put((rank, layer.col0, layer.ldy, err, outs, None))
    except Exception as exc:  # reported to the parent, which fails the test
        q.put((rank, None, None, None, None, repr(exc)))
    finally:
        dist.destroy_process_group()


def test_tp_two_processes_over_ipc_on_one_gpu():
    fmt, widths, K, Ms, seed = "fp8_dynamic", [384, 256], 1024, [3, 16, 1], 21
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_rank, args=(r, 2, port, fmt, widths, K, Ms, seed, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted([q.get(timeout=300) for _ in procs], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=120)
    for rank, col0, ldy, err, outs, exc in results:
        assert exc is None, f"rank {rank}: {exc}"
        assert col0 == sum(widths[:rank]) and ldy == sum(widths) and err == 0
    w = synth.weights(sum(widths), K, seed)
    for call, M in enumerate(Ms):
        x = synth.activations(M, K, seed + 7 * call)
        yref, bound = oracle_layer(fmt, x, w)
        for rank, _, _, _, outs, _ in results:
            check_layer(fmt, outs[call].view(torch.bfloat16), yref, bound, K, f"IPC rank {rank} call {call}")
    for p in procs:
        assert p.exitcode == 0
