"""R expert-parallel ranks in one process, one thread per rank (test infrastructure).

``LoopbackComm`` implements the collectives of ``MoeEP`` by copying between the ranks' tensors:
for the all-to-all (split along dim 0, block s of the output from source s) and the all-gather,
every rank deposits its input, waits for all ranks on a host barrier, copies from every source, and
waits again before its input can be overwritten; ``alloc_shared`` hands every rank the other ranks'
buffers themselves (one address space: the peer-memory exchange reads and writes them directly).  On one GPU, all threads issue their work to the same (default) stream, so the
copies run after every rank's producing kernels and before any later overwrite: no kernel ever
waits on another.
"""
import threading

import torch


class LoopbackHub:
    def __init__(self, R: int):
        self.R = R
        self.barrier = threading.Barrier(R, timeout=120)
        self.slots = [None] * R


class LoopbackComm:
    def __init__(self, hub: LoopbackHub, rank: int):
        self.hub, self.rank, self.size = hub, rank, hub.R

    def all_to_all(self, out, inp, out_splits=None, in_splits=None):
        hub, R = self.hub, self.hub.R
        if in_splits is None:
            in_splits = [inp.shape[0] // R] * R
        hub.slots[self.rank] = (inp, list(in_splits))
        hub.barrier.wait()
        pos = 0
        for s in range(R):
            src, splits = hub.slots[s]
            lo, n = sum(splits[:self.rank]), splits[self.rank]
            if out_splits is not None:
                assert out_splits[s] == n, (out_splits, s, n)
            out[pos:pos + n].copy_(src[lo:lo + n])
            pos += n
        hub.barrier.wait()


    def all_gather(self, out, inp):
        hub, R = self.hub, self.hub.R
        hub.slots[self.rank] = inp
        hub.barrier.wait()
        n = inp.shape[0]
        for s in range(R):
            out[s * n:(s + 1) * n].copy_(hub.slots[s])
        hub.barrier.wait()

    def barrier(self, device=None):
        self.hub.barrier.wait()

    def alloc_shared(self, shape, dtype, device):
        """Every rank allocates its own buffer; all ranks see all of them (one address space)."""
        hub = self.hub
        t = torch.empty(shape, dtype=dtype, device=device)
        hub.slots[self.rank] = t
        hub.barrier.wait()
        peers = list(hub.slots)
        hub.barrier.wait()
        return t, peers


def run_ranks(R: int, fn):
    """fn(rank, comm) on R threads; returns the per-rank results, re-raising the first error."""
    hub = LoopbackHub(R)
    res, errs = [None] * R, []

    def body(r):
        try:
            res[r] = fn(r, LoopbackComm(hub, r))
        except BaseException as e:  # noqa: BLE001 - reported below
            errs.append(e)
            hub.barrier.abort()

    ts = [threading.Thread(target=body, args=(r,)) for r in range(R)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    if errs:
        raise errs[0]
    return res
