"""Data-parallel exchange of the packed skew-parameter gradients, overlapped with the backward pass.

POET-X trains under plain data parallelism (agidaily.cc article, the distributed-training
paragraph; replication review, "Weaknesses": the DDP runs behind the Table 10 scaling): every
rank holds a replica of the frozen W0', of theta and of the permutations, runs the layer step on
its own tokens, and the only exchange is the sum of the packed gradients d theta over the ranks.
Only the packed form moves: b(b-1)/2 floats per block.

GradBuckets keeps every layer's gradient (theta_R then theta_P, as poetx_backward writes them) as
a contiguous slice of one flat buffer laid out in forward order.  The backward pass visits the
layers in reverse, so the layers it finishes one after another are neighbours in memory: a bucket
is a run of consecutive layers (about bucket_bytes), reduced in place with one asynchronous
all-reduce as soon as its last layer's backward has been enqueued.  With NCCL the collective is
ordered after everything the caller's stream holds at that moment and runs beside the backward of
the layers below; finish() makes the caller's stream wait for all of them.  With gloo (CPU
tensors) the same calls run on the host.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple


def plan_buckets(sizes: Sequence[int], bucket_bytes: int, elem_bytes: int = 4) -> List[Tuple[int, int]]:
    """Buckets as (first_layer, last_layer + 1), in the order the backward pass completes them
    (last layers first).  Each bucket is a run of consecutive layers whose packed gradients add up
    to at least bucket_bytes (the last one may be smaller); every layer is in exactly one bucket."""
    if bucket_bytes <= 0:
        raise ValueError("bucket_bytes must be positive")
    buckets = []
    end = len(sizes)
    acc = 0
    for i in range(len(sizes) - 1, -1, -1):
        acc += sizes[i] * elem_bytes
        if acc >= bucket_bytes or i == 0:
            buckets.append((i, end))
            end, acc = i, 0
    return buckets


class GradBuckets:
    """Sums a flat packed-gradient buffer over the ranks of `group`, bucket by bucket, while the
    backward pass is still running.

    flat:   1-D float32 tensor holding every layer's packed gradient, layer i at
            [offsets[i], offsets[i + 1]) (forward order).
    sizes:  number of packed parameters of each layer (both sides), in forward order.

    Per step: call layer_done(i) right after enqueuing layer i's backward (layers in reverse
    order, each exactly once), then finish() before anything reads the summed gradients.
    """

    def __init__(self, flat, sizes: Sequence[int], bucket_bytes: int = 25 << 20, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.flat = flat
        self.sizes = list(sizes)
        self.offsets = [0]
        for n in self.sizes:
            self.offsets.append(self.offsets[-1] + n)
        if self.offsets[-1] > flat.numel():
            raise ValueError("the flat buffer is smaller than the layers' packed gradients")
        self.group = group
        self.buckets = plan_buckets(self.sizes, bucket_bytes, flat.element_size())
        self.bucket_of = {}
        for bi, (lo, hi) in enumerate(self.buckets):
            for layer in range(lo, hi):
                self.bucket_of[layer] = bi
        self._reset()

    def _reset(self):
        self.pending = [hi - lo for lo, hi in self.buckets]
        self.handles = []
        self.launched = []  # bucket indices in launch order (kept for inspection)

    def layer_done(self, layer: int) -> None:
        bi = self.bucket_of[layer]
        self.pending[bi] -= 1
        if self.pending[bi] < 0:
            raise RuntimeError(f"layer {layer} reported twice in one step")
        if self.pending[bi] == 0:
            lo, hi = self.buckets[bi]
            view = self.flat[self.offsets[lo]:self.offsets[hi]]
            self.handles.append(self.dist.all_reduce(view, op=self.dist.ReduceOp.SUM, group=self.group,
                                                     async_op=True))
            self.launched.append(bi)

    def finish(self) -> None:
        """Waits for every bucket (the caller's CUDA stream waits for NCCL; gloo blocks the host)
        and re-arms for the next step.  Every layer must have been reported."""
        if any(p != 0 for p in self.pending):
            raise RuntimeError("finish() before every layer's backward was reported")
        for h in self.handles:
            h.wait()
        self._reset()
