"""A quantized linear layer built on the C ABI, with the method's hybrid
dispatch: token counts up to 32 replay a CUDA graph captured once per M
bucket (1, 2, 4, 8, 16, 24, 32); larger counts launch directly.

Hybrid dispatch and graph replay follow "Building a High-Performance and
Portable vLLM Linear Backend with Helion", section "Hybrid dispatch"
("Despacho hibrido"): small shapes run under CUDA-graph replay so the CPU's
launch cost does not eat the kernel's gain.
"""
from __future__ import annotations

import torch

import quantized_gemm_decode_b200 as qgd

DECODE_BUCKETS = (1, 2, 4, 8, 16, 24, 32)
GRAPH_MAX_M = 32

_FMT = {"fp8_dynamic": qgd.FMT_FP8_DYNAMIC, "w8a8_int8": qgd.FMT_W8A8_INT8, "block_fp8": qgd.FMT_BLOCK_FP8}


class QuantizedLinear:
    """y = x @ W^T with W quantized once at construction and x quantized
    dynamically on every call, both by this library's kernels."""

    def __init__(self, w: torch.Tensor, fmt: str = "fp8_dynamic", wq=None, sw=None):
        if fmt not in _FMT:
            raise ValueError(f"unknown format {fmt}")
        self.fmt = fmt
        self.fmt_id = _FMT[fmt]
        self.N, self.K = (w.shape if w is not None else wq.shape)
        self.device = (w if w is not None else wq).device
        if wq is None:
            if fmt == "block_fp8":
                wq, sw = qgd.quant_weight_block128(w)
            else:
                qt = qgd.QTYPE_INT8 if fmt == "w8a8_int8" else qgd.QTYPE_E4M3
                wq, sw = qgd.quant_weight_per_channel(w, qt)
        self.wq, self.sw = wq, sw
        need = max(max(qgd.qgd_workspace_size(self.fmt_id, m, self.N, self.K),
                       qgd.qgd_layer_workspace_size(self.fmt_id, m, self.N, self.K)) for m in DECODE_BUCKETS)
        self.ws = qgd.Workspace(need, self.device)
        self._graphs: dict = {}

    # ---- eager path ---------------------------------------------------
    def quantize(self, x: torch.Tensor, xq=None, sx=None):
        if self.fmt == "block_fp8":
            return qgd.quant_act_group128(x, xq=xq, sx=sx)
        qt = qgd.QTYPE_INT8 if self.fmt == "w8a8_int8" else qgd.QTYPE_E4M3
        return qgd.quant_act_per_token(x, qt, xq=xq, sx=sx)

    def gemm(self, xq, sx, y=None):
        fn = {"fp8_dynamic": qgd.qlinear_fp8_dynamic, "w8a8_int8": qgd.qlinear_w8a8_int8,
              "block_fp8": qgd.qlinear_block_fp8}[self.fmt]
        self.ws.ensure(qgd.qgd_workspace_size(self.fmt_id, xq.shape[0], self.N, self.K))
        return fn(xq, sx, self.wq, self.sw, y=y, ws=self.ws)

    def layer(self, x: torch.Tensor, y=None) -> torch.Tensor:
        """The whole layer call from bf16 x (possibly a column slice of a
        wider matrix): quantization and GEMM, fused into one kernel when the
        layer plan says so."""
        self.ws.ensure(qgd.qgd_layer_workspace_size(self.fmt_id, x.shape[0], self.N, self.K))
        return qgd.qlinear_bf16(self.fmt_id, x, self.wq, self.sw, y=y, ws=self.ws)

    def forward_eager(self, x: torch.Tensor, y=None) -> torch.Tensor:
        return self.layer(x, y=y)

    # ---- graph path ---------------------------------------------------
    def capture(self, buckets=DECODE_BUCKETS) -> None:
        """Capture one graph per M bucket (static input/output buffers)."""
        for mb in buckets:
            x = torch.zeros((mb, self.K), dtype=torch.bfloat16, device=self.device)
            y = torch.empty((mb, self.N), dtype=torch.bfloat16, device=self.device)
            xq = torch.empty((mb, self.K), dtype=torch.int8 if self.fmt == "w8a8_int8" else torch.float8_e4m3fn,
                             device=self.device)
            sx = torch.empty((mb, self.K // 128) if self.fmt == "block_fp8" else (mb,), dtype=torch.float32,
                             device=self.device)
            self.ws.ensure(qgd.qgd_layer_workspace_size(self.fmt_id, mb, self.N, self.K))
            s = torch.cuda.Stream(self.device)
            s.wait_stream(torch.cuda.current_stream(self.device))
            with torch.cuda.stream(s):
                self.layer(x, y)
            torch.cuda.current_stream(self.device).wait_stream(s)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.layer(x, y)
            self._graphs[mb] = (g, x, y)

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        """Apply the layer.  M <= 32 replays the captured graph of M's bucket
        (inputs are copied into its static buffer; x may live on the host,
        pinned); larger M runs eagerly.  With `out` (possibly pinned host
        memory) the result is copied there and `out` is returned."""
        M = x.shape[0]
        if M <= GRAPH_MAX_M and self._graphs:
            mb = qgd.qgd_m_bucket(M)
            g, xs, ys = self._graphs[mb]
            xs[:M].copy_(x, non_blocking=True)
            g.replay()
            if out is not None:
                out.copy_(ys[:M], non_blocking=True)
                return out
            return ys[:M]
        xd = x if x.is_cuda else x.to(self.device, non_blocking=True)
        y = self.forward_eager(xd)
        if out is not None:
            out.copy_(y, non_blocking=True)
            return out
        return y


class DecodeStep:
    """One decode step of several quantized linear layers captured as a single
    CUDA graph, host I/O included: each layer's activations are copied from
    pinned host memory on a copy stream (all copies issued up front), each
    layer quantizes and multiplies on the compute stream as soon as its input
    has landed, and each result is copied back to pinned host memory on a
    second copy stream while the next layers compute.

    `calls` is a list of (layer, M); `x_host[i]` / `y_host[i]` are pinned
    host tensors of shape [M, K] / [M, N].  replay() runs the whole step
    asynchronously on the current stream; synchronize before reading y_host.

    `join_every` groups the input copies: the compute stream waits once per
    group of that many layers (for all of the group's copies) instead of once
    per layer.  Every such wait is a dependency on a copy in the middle of the
    chain of kernels, where the next kernel can no longer be launched early
    behind the one before it.  On B200, over the 28 layers of the 8B-class
    FP8 sweep, one wait per 4 layers was fastest (0.49 ms per step against
    0.54 ms for one per layer and 0.63 ms for a single wait up front).
    `out_every` likewise groups the result copies (one fork of the compute
    stream per group of that many layers); per layer measured fastest (0.49
    ms against 0.50-0.55 ms for groups of 2-7).
    """

    def __init__(self, calls, x_host, y_host, join_every: int = 4, out_every: int = 1):
        self.join_every = max(1, int(join_every))
        self.out_every = max(1, int(out_every))
        self.calls = list(calls)
        dev = self.calls[0][0].device
        self.x_dev, self.y_dev = [], []
        for (layer, M) in self.calls:
            self.x_dev.append(torch.empty((M, layer.K), dtype=torch.bfloat16, device=dev))
            self.y_dev.append(torch.empty((M, layer.N), dtype=torch.bfloat16, device=dev))
            layer.ws.ensure(qgd.qgd_layer_workspace_size(layer.fmt_id, M, layer.N, layer.K))
        self.x_host, self.y_host = list(x_host), list(y_host)
        self.graph = torch.cuda.CUDAGraph()
        main = torch.cuda.Stream(dev)
        copy_in = torch.cuda.Stream(dev)
        copy_out = torch.cuda.Stream(dev)
        # warm up outside capture (loads the kernels, sizes the workspaces)
        with torch.cuda.stream(main):
            self._body(main, None, None)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(self.graph, stream=main):
            self._body(main, copy_in, copy_out)

    def _body(self, main, copy_in, copy_out):
        if copy_in is None:
            for i, (layer, M) in enumerate(self.calls):
                self.x_dev[i].copy_(self.x_host[i], non_blocking=True)
                layer.layer(self.x_dev[i], self.y_dev[i])
                self.y_host[i].copy_(self.y_dev[i], non_blocking=True)
            return
        landed = {}
        copy_in.wait_stream(main)
        copy_out.wait_stream(main)
        n = len(self.calls)
        with torch.cuda.stream(copy_in):
            for i in range(n):
                self.x_dev[i].copy_(self.x_host[i], non_blocking=True)
                if (i + 1) % self.join_every == 0 or i == n - 1:
                    ev = torch.cuda.Event()
                    ev.record(copy_in)
                    landed[i // self.join_every] = ev
        for i, (layer, M) in enumerate(self.calls):
            if i % self.join_every == 0:
                main.wait_event(landed[i // self.join_every])
            layer.layer(self.x_dev[i], self.y_dev[i])
            # results leave in groups too: one fork from the compute stream per group
            if (i + 1) % self.out_every == 0 or i == n - 1:
                done = torch.cuda.Event()
                done.record(main)
                copy_out.wait_event(done)
                with torch.cuda.stream(copy_out):
                    for k in range(i - (i % self.out_every), i + 1):
                        self.y_host[k].copy_(self.y_dev[k], non_blocking=True)
        main.wait_stream(copy_in)
        main.wait_stream(copy_out)

    def replay(self):
        self.graph.replay()


# The four projections of one dense decoder layer and where each one's input
# comes from: (name, source, input columns).  source -1 is the chain input;
# otherwise the input is the first `input columns` columns of that earlier
# projection's output.  The o projection reads the first 4096 columns of
# qkv's output and down the first 12288 of gate_up's: in the model, attention
# and the gated activation sit there, and here a column slice of the right
# width stands in for each (neither is part of the linear layer's path).
LAYER_8B = (("qkv", -1, 4096), ("o", 0, 4096), ("gate_up", 1, 4096), ("down", 2, 12288))


class DecodeChain:
    """Dependent linear layers of one decode step, captured as one CUDA graph
    per token count: each layer call quantizes its input -- a column slice of
    an earlier layer's bf16 output, read in place through the row stride --
    and runs its GEMM (one fused kernel when the layer plan says so), so every
    kernel waits for the one before it (the conditions of a model's forward
    pass, unlike independent calls).

    `layers` is a list of QuantizedLinear in chain order; `wiring` a list of
    (name, source, columns) as LAYER_8B.  capture(M) builds the graph for M
    tokens; run(M, x) copies x into the chain input and replays it; outputs(M)
    are the layers' bf16 outputs and inputs(M) the bf16 inputs they read.
    """

    def __init__(self, layers, wiring=LAYER_8B):
        if len(layers) != len(wiring):
            raise ValueError("one wiring entry per layer")
        self.layers = list(layers)
        self.wiring = list(wiring)
        self.device = self.layers[0].device
        for i, (layer, (_, src, cols)) in enumerate(zip(self.layers, self.wiring)):
            width = self.layers[0].K if src < 0 else self.layers[src].N
            if src >= i or cols != layer.K or cols > width:
                raise ValueError(f"layer {i}: input of {cols} columns from source {src} does not fit")
        self._bufs: dict = {}
        self._graphs: dict = {}

    def _buffers(self, M: int):
        if M not in self._bufs:
            x = torch.zeros((M, self.layers[0].K), dtype=torch.bfloat16, device=self.device)
            ys = []
            for layer in self.layers:
                ys.append(torch.empty((M, layer.N), dtype=torch.bfloat16, device=self.device))
                layer.ws.ensure(qgd.qgd_layer_workspace_size(layer.fmt_id, M, layer.N, layer.K))
            self._bufs[M] = (x, ys)
        return self._bufs[M]

    def _input(self, M: int, i: int) -> torch.Tensor:
        x, ys = self._buffers(M)
        _, src, cols = self.wiring[i]
        return x if src < 0 else ys[src][:, :cols]

    def _body(self, M: int):
        _, ys = self._buffers(M)
        for i, layer in enumerate(self.layers):
            layer.layer(self._input(M, i), ys[i])

    def capture(self, M: int) -> None:
        self._buffers(M)
        s = torch.cuda.Stream(self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            self._body(M)  # warm-up outside capture
        torch.cuda.current_stream(self.device).wait_stream(s)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self._body(M)
        self._graphs[M] = g

    def graph(self, M: int) -> torch.cuda.CUDAGraph:
        if M not in self._graphs:
            self.capture(M)
        return self._graphs[M]

    def run(self, M: int, x: torch.Tensor | None = None) -> torch.Tensor:
        """Replay the chain for M tokens (after copying x into its input) and
        return the last layer's output buffer."""
        g = self.graph(M)
        if x is not None:
            self._bufs[M][0].copy_(x, non_blocking=True)
        g.replay()
        return self._bufs[M][1][-1]

    def input_buffer(self, M: int) -> torch.Tensor:
        return self._buffers(M)[0]

    def outputs(self, M: int) -> list:
        return self._buffers(M)[1]

    def inputs(self, M: int) -> list:
        """The bf16 input each layer quantized (views into earlier outputs)."""
        return [self._input(M, i) for i in range(len(self.layers))]


# ---------------------------------------------------------------------------
# Column-parallel (tensor-parallel) layer
# ---------------------------------------------------------------------------
_TP_FMT = {"fp8_dynamic": qgd.FMT_FP8_DYNAMIC, "w8a8_int8": qgd.FMT_W8A8_INT8, "block_fp8": qgd.FMT_BLOCK_FP8,
           "mxfp8": qgd.FMT_MXFP8, "nvfp4": qgd.FMT_NVFP4}


def quantize_weight(w: torch.Tensor, fmt: str) -> tuple:
    """(wq, sw, sw_block) of a bf16 weight [N, K] in a layer format, as the
    layer calls take them (sw_block: the NVFP4 E4M3 block scales, else None)."""
    if fmt == "block_fp8":
        wq, sw = qgd.quant_weight_block128(w)
        return wq, sw, None
    if fmt == "mxfp8":
        wq, sw = qgd.quant_mx(w)
        return wq, sw, None
    if fmt == "nvfp4":
        wq, sb, g = qgd.quant_nv(w)
        return wq, g, sb
    qt = qgd.QTYPE_INT8 if fmt == "w8a8_int8" else qgd.QTYPE_E4M3
    wq, sw = qgd.quant_weight_per_channel(w, qt)
    return wq, sw, None


class _LibraryIpc:
    malloc = staticmethod(qgd.ipc_malloc)
    open = staticmethod(qgd.ipc_open)
    close = staticmethod(qgd.ipc_close)
    free = staticmethod(qgd.ipc_free)


def _align(n: int, a: int = 256) -> int:
    return (n + a - 1) // a * a


class ColumnParallelLinear:
    """y = x @ W^T with W's rows (the output columns) split over the ranks of
    a torch.distributed group, one GPU per rank, and the all-gather of y fused
    into the GEMM: each rank's kernel stores its columns straight into every
    rank's full output over peer memory (NVLink) and then raises one flag per
    rank, so every rank ends the call holding all of y.

    Each rank owns one shared device buffer, mapped by all ranks (CUDA IPC):
    two full outputs [max_m, ldy] bf16 (successive calls alternate, so that a
    rank already running its next call never overwrites the output another
    rank is still reading) and a flag array of one uint32 per rank plus this
    rank's call counter, which the kernels advance (so a captured graph of the
    calls stays in step).  Shards may differ in width; col0 and ldy come from
    an all-gather of the widths.
    """

    def __init__(self, w_shard: torch.Tensor | None, fmt: str = "fp8_dynamic", group=None, max_m: int = 32,
                 weights: tuple | None = None, ipc=None):
        import torch.distributed as dist

        if fmt not in _TP_FMT:
            raise ValueError(f"unknown format {fmt}")
        self.fmt, self.fmt_id = fmt, _TP_FMT[fmt]
        self.group = group
        self._dist = dist if dist.is_available() and dist.is_initialized() else None
        self.G = self._dist.get_world_size(group) if self._dist else 1
        self.rank = self._dist.get_rank(group) if self._dist else 0
        if self.G > qgd.MAX_TP_RANKS:
            raise ValueError(f"at most {qgd.MAX_TP_RANKS} ranks share one output")
        self.wq, self.sw, self.sw_block = weights if weights is not None else quantize_weight(w_shard, fmt)
        self.N = self.wq.shape[0]
        self.K = self.wq.shape[1] * (2 if fmt == "nvfp4" else 1)
        self.device = self.wq.device
        widths = self._all_gather(self.N)
        self.col0, self.ldy = sum(widths[:self.rank]), sum(widths)
        self.max_m = max_m
        self.out_bytes = max_m * self.ldy * 2
        self.flags_off = 2 * _align(self.out_bytes)
        self.nbytes = self.flags_off + _align(4 * (self.G + 1))
        self._ipc = ipc if ipc is not None else _LibraryIpc
        self.own, handle = self._ipc.malloc(self.nbytes)
        handles = self._all_gather(handle)
        self.bases = [self.own if r == self.rank else self._ipc.open(handles[r]) for r in range(self.G)]
        self.ws = qgd.Workspace(qgd.qgd_tp_workspace_size(self.fmt_id, max_m, self.N, self.K), self.device)
        self.calls = 0

    def _all_gather(self, obj) -> list:
        if self._dist is None:
            return [obj]
        out = [None] * self.G
        self._dist.all_gather_object(out, obj, group=self.group)
        return out

    def output_ptr(self, rank: int, buf: int) -> int:
        return self.bases[rank] + buf * _align(self.out_bytes)

    def flags_ptr(self, rank: int) -> int:
        return self.bases[rank] + self.flags_off

    def launch(self, x: torch.Tensor, stream=None) -> int:
        """Enqueue this rank's share of the call; returns the output buffer
        (0 or 1) it writes.  Every rank must launch the same sequence of calls."""
        M = x.shape[0]
        if M > self.max_m:
            raise ValueError(f"M={M} exceeds the buffers' {self.max_m} rows")
        buf = self.calls & 1
        self.calls += 1
        if M == 0:
            return buf
        qgd.qlinear_tp_bf16(self.fmt_id, x, self.wq, self.sw, self.sw_block, ranks=self.G, rank=self.rank,
                            col0=self.col0, ldy=self.ldy, ys=[self.output_ptr(r, buf) for r in range(self.G)],
                            flags=[self.flags_ptr(r) for r in range(self.G)], ws=self.ws, stream=stream)
        return buf

    def wait(self, M: int, buf: int, stream=None) -> torch.Tensor:
        """Enqueue the wait for every rank's share of the last call and return
        the full output [M, ldy] (a view of this rank's shared buffer, valid
        until the call after next)."""
        if M > 0:
            qgd.qgd_tp_wait(self.flags_ptr(self.rank), self.G, stream=stream)
        full = qgd.tensor_at(self.output_ptr(self.rank, buf), (self.max_m, self.ldy), torch.bfloat16, self.device)
        return full[:M]

    def __call__(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        buf = self.launch(x, stream=stream)
        return self.wait(x.shape[0], buf, stream=stream)

    def close(self) -> None:
        """Unmap the peers' buffers and free this rank's (collective: every
        rank calls it, after its last use of the outputs)."""
        if self.bases is None:
            return
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        if self._dist is not None:
            self._dist.barrier(group=self.group)  # no rank still writes into another's buffer
        for r, p in enumerate(self.bases):
            if r != self.rank:
                self._ipc.close(p)
        if self._dist is not None:
            self._dist.barrier(group=self.group)  # every mapping of this rank's buffer is gone
        self._ipc.free(self.own)
        self.bases = None
