"""Row-sharded fused product over several GPUs, one process per GPU.

Each rank decodes and multiplies its own contiguous range of a layer's rows, and one all-gather
over the process group assembles y on every rank.  The pages give only the motivation: the fused
kernel streams the packed weights once and never writes dequantized weights back
(papernotes.org notes, 关键设计 4), so splitting the rows over G GPUs splits that stream G ways
and leaves a single exchange, the output vector (4 bytes per row and batch row).

This module is host logic only: the row partition, the local weight view (a row slice of the
packed words and gains, no copy) and the gather.  The product itself is llvq_gemv /
llvq_gemm_smallbatch on the local rows, and the gather is torch.distributed's all-gather (NCCL
between GPUs).  Slices are padded to the largest one, because NCCL's all-gather takes equal sizes.
"""
from __future__ import annotations


def row_ranges(rows: int, world: int) -> list[tuple[int, int]]:
    """Contiguous [r0, r1) per rank covering 0..rows; the first rows % world ranks take one row
    more than the others."""
    if rows < 0 or world < 1:
        raise ValueError("rows >= 0 and world >= 1")
    base, extra = divmod(rows, world)
    out, r0 = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((r0, r0 + n))
        r0 += n
    return out


def gather_rows(y_local, rows: int, world: int, group=None):
    """All-gather each rank's outputs y_local [batch, r1 - r0] into y [batch, rows] on every rank
    (ranks in order; the padding of the shorter slices dropped)."""
    import torch
    import torch.distributed as dist
    ranges = row_ranges(rows, world)
    width = max(r1 - r0 for r0, r1 in ranges)
    buf = y_local.new_zeros((y_local.shape[0], width))
    buf[:, : y_local.shape[1]] = y_local
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf, group=group)
    return torch.cat([p[:, : r1 - r0] for p, (r0, r1) in zip(parts, ranges)], dim=1)


class RowShardedProduct:
    """y = W x for a layer whose rows are split over the ranks of a process group.

    words / gains: this process's full-layer tensors on its GPU ([rows, ...], row-major; only the
    local rows are read), or only the local rows when local=True.  Every rank calls the product
    with the same activations and gets the whole y."""

    def __init__(self, codec, words, gains, rows: int, cols: int, gain_mode: int, row_pitch_words: int,
                 rank: int, world: int, group=None, local: bool = False):
        self.codec, self.rows, self.rank, self.world, self.group = codec, rows, rank, world, group
        self.r0, self.r1 = row_ranges(rows, world)[rank]
        if not local:
            words, gains = words[self.r0:self.r1], gains[self.r0:self.r1]
        self.weight = codec.weight(words, gains, self.r1 - self.r0, cols, gain_mode, row_pitch_words)
        self._keep = (words, gains)

    def local(self, X, Y_local, batch: int = 1, stream=None):
        """This rank's rows only: Y_local [batch, r1 - r0] (fp32, on the GPU)."""
        if self.r1 == self.r0:
            return Y_local
        if batch == 1:
            self.codec.gemv(self.weight, X, Y_local, stream=stream)
        else:
            self.codec.gemm(self.weight, X, Y_local, batch, stream=stream)
        return Y_local

    def __call__(self, X, Y_local, batch: int = 1, stream=None):
        """The whole y [batch, rows] on every rank: the local product, then the all-gather (on the
        current stream, which first waits for `stream` when the product ran there)."""
        self.local(X, Y_local, batch, stream)
        if stream is not None:
            import torch
            torch.cuda.current_stream().wait_stream(stream)
        return gather_rows(Y_local, self.rows, self.world, self.group)
