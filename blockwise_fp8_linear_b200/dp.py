"""Data-parallel exchange of the FP32 main gradients of the FP8 linear layers.

Puro-2B (part 3/7, section 3.1) trains data-parallel: every rank runs the same layers
on its own micro-batches, and the weight gradients are summed over the ranks before
the optimizer step.  The reading notes on the paper (section 2.3, the FP8 table) keep
gradient accumulation in FP32.  Here each rank's wgrad accumulates into an FP32 main
gradient with fp8_gemm_wgrad_acc32 (the token reduction of its own shard), and this
module sums those FP32 buffers over the ranks with a reduce-scatter: rank r keeps rows
[r*out/N, (r+1)*out/N) of every dW[out][in], the layout of an optimizer sharded by
rows.  The sum over ranks is the wgrad over the concatenated token shards, because
the token-dim quantization groups (128 tokens) never straddle a shard boundary when
each shard is a multiple of 128 tokens.

The collective is torch.distributed's reduce_scatter_tensor: NCCL over NVLink on GPUs
(issued on the stream that produced the gradient, so it overlaps later kernels), gloo
on CPU for the tests.  It is a library collective, not a fused GEMM + reduce-scatter
kernel; no load with cluster multicast is involved.
"""
from __future__ import annotations


class DpGradReducer:
    """Reduce-scatter of one FP32 main gradient per linear layer.

    shapes: (out_features, in_features) per linear; out_features must be divisible by
    the world size.  launch(i, dw32, stream) enqueues the sum of linear i's dw32 over
    the ranks (asynchronously; on `stream` if given); wait() blocks until every
    launched exchange is done (on GPUs: makes the current stream wait).  shards[i]
    then holds this rank's rows of the summed gradient."""

    def __init__(self, shapes, world: int, device, dtype=None):
        import torch
        self.world = int(world)
        self.dtype = torch.float32 if dtype is None else dtype
        for dout, din in shapes:
            if dout % self.world:
                raise ValueError(f"out_features {dout} is not divisible by the world size {world}")
        self.shapes = [(int(dout), int(din)) for dout, din in shapes]
        self.shards = [torch.empty(dout // self.world, din, dtype=self.dtype, device=device)
                       for dout, din in self.shapes]
        self.pending = []

    @staticmethod
    def rows(dout: int, world: int, rank: int):
        """Rows [lo, hi) of a dW[dout][din] that rank `rank` keeps."""
        return rank * dout // world, (rank + 1) * dout // world

    def launch(self, i: int, dw, stream=None):
        import torch
        import torch.distributed as dist
        dout, din = self.shapes[i]
        if tuple(dw.shape) != (dout, din) or dw.dtype != self.dtype or not dw.is_contiguous():
            raise ValueError(f"gradient {i} must be a contiguous {self.dtype} [{dout}][{din}] tensor")
        if stream is not None:
            with torch.cuda.stream(stream):
                h = dist.reduce_scatter_tensor(self.shards[i], dw, op=dist.ReduceOp.SUM,
                                               async_op=True)
        else:
            h = dist.reduce_scatter_tensor(self.shards[i], dw, op=dist.ReduceOp.SUM, async_op=True)
        self.pending.append(h)

    def wait(self):
        for h in self.pending:
            h.wait()
        self.pending.clear()
