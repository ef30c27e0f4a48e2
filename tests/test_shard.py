"""The row-sharded product's host logic on CPU (codebook_free_lattice_b200/shard.py): the row
partition, and two or three gloo ranks, as under torchrun, each computing its own rows and
gathering y.  The per-rank product is the CPU oracle's fp64 product on the rank's rows, through a
stand-in codec with the binding's weight/gemv/gemm calls, so that the slicing, the local product
and the gather run end to end without a GPU; every rank must end with the oracle's product of
the whole layer.  (On GPUs the same class calls llvq_gemv / llvq_gemm_smallbatch and the
gather runs over NCCL; this run has one GPU, so that is not exercised here.)
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist                           # noqa: E402
import torch.multiprocessing as mp                         # noqa: E402

from codebook_free_lattice_b200.shard import row_ranges   # noqa: E402


@pytest.mark.parametrize("rows,world", [(37, 2), (37, 3), (4096, 8), (5, 8), (0, 2), (24, 1)])
def test_row_ranges_cover_contiguously(rows, world):
    rr = row_ranges(rows, world)
    assert len(rr) == world and rr[0][0] == 0 and rr[-1][1] == rows
    assert all(a[1] == b[0] for a, b in zip(rr, rr[1:]))
    sizes = [r1 - r0 for r0, r1 in rr]
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def layer(rows=37, cols=96, batch=2, seed=5):
    import oracle
    from codebook_free_lattice_b200 import synth
    o = oracle.Codec(48)
    nb = cols // 24
    lo, _ = synth.uniform_indices(synth.rng(seed, 0), rows * nb, o.n_points, 48)
    codes = synth.gain_codes(synth.rng(seed, 1), rows * nb)
    words = synth.pack_words(lo, None, codes, 48).reshape(rows, nb)
    gains = synth.chi24_tables(synth.rng(seed, 2), rows)
    x = synth.activations(synth.rng(seed, 3), batch, cols)
    return o, words, gains, x, nb


class OracleCodec:
    """The binding's weight/gemv/gemm calls, computed by the CPU oracle on CPU tensors."""

    def __init__(self, o, nb):
        self.o, self.nb = o, nb

    def weight(self, words, gains, rows, cols, gain_mode, pitch):
        return (words.numpy(), gains.numpy(), rows, gain_mode)

    def gemv(self, w, X, Y, stream=None):
        self.gemm(w, X, Y, 1)

    def gemm(self, w, X, Y, batch, stream=None):
        words, gains, rows, mode = w
        y = self.o.gemm(words.view(np.uint64), self.nb, mode, gains.view(np.uint16), X.numpy(), batch)
        Y.copy_(torch.from_numpy(y).reshape(batch, rows))


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from codebook_free_lattice_b200.shard import RowShardedProduct
        o, words, gains, x, nb = layer()
        rows, cols, batch = words.shape[0], nb * 24, x.shape[0]
        prod = RowShardedProduct(OracleCodec(o, nb), torch.from_numpy(words.view(np.int64)),
                                 torch.from_numpy(gains.view(np.int16)), rows, cols, 1, nb, rank, world)
        Y_local = torch.empty((batch, prod.r1 - prod.r0), dtype=torch.float64)
        y = prod(torch.from_numpy(x.view(np.int16)), Y_local, batch)
        dist.barrier()
        q.put((rank, prod.r0, prod.r1, y.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_gather_the_whole_product(world):
    port = socket.socket()
    port.bind(("127.0.0.1", 0))
    p = port.getsockname()[1]
    port.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, p, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    out = sorted((q.get(timeout=120) for _ in range(world)), key=lambda t: t[0])
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    o, words, gains, x, nb = layer()
    ref = o.gemm(words, nb, 1, gains, x, x.shape[0])
    assert [(r0, r1) for _, r0, r1, _ in out] == row_ranges(words.shape[0], world)
    for _, _, _, y in out:
        assert np.array_equal(y, ref)
