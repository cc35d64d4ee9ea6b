"""Host logic of the expert-parallel layer on CPU (gloo, world size 2): the pointer-table
exchange (each rank's own buffers by address, a peer's through one mapping per peer
allocation) and the all-gather of the count vectors in rank order."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from load_balanced_dispatch_warp_b200 import ep


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class FakeBuf:
    """Stands in for a device tensor: an address inside a numbered allocation."""

    def __init__(self, alloc, offset, base=1 << 40):
        self.alloc, self.offset, self.base = alloc, offset, base

    def data_ptr(self):
        return self.base + self.alloc * (1 << 30) + self.offset


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        comm = ep.GlooComm()
        assert (comm.rank, comm.world) == (rank, world)
        # recv and y share allocation 0 of this rank, the weights sit in allocation 1
        local = {"recv": FakeBuf(0, 0), "y": FakeBuf(0, 4096), "W1": FakeBuf(1, 0),
                 "W3": FakeBuf(1, 8192), "W2": FakeBuf(1, 16384)}
        opened = []

        def export(t):
            return (f"rank{rank}-alloc{t.alloc}".encode().ljust(64, b"\0"), t.offset)

        def import_base(handle):
            opened.append(handle)
            name = handle.rstrip(b"\0").decode()
            r, a = name.split("-")
            return 7 << 44 | int(r[4:]) << 36 | int(a[5:]) << 30

        tables, bases = ep.exchange_pointers(local, rank, world, comm._gather_objects, export,
                                             import_base)
        send = torch.arange(5, dtype=torch.int32) + 100 * rank
        gathered = torch.zeros(world, 5, dtype=torch.int32)
        comm.all_gather(send, gathered)
        comm.barrier()
        out[rank] = (tables, len(bases), len(opened), gathered.tolist())
    finally:
        dist.destroy_process_group()


def test_pointer_tables_and_gather_two_ranks():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        tables, nbases, nopened, gathered = out[rank]
        peer = 1 - rank
        # each peer allocation mapped once: recv+y share one, the weights another
        assert nbases == 2 and nopened == 2
        assert gathered == [[0, 1, 2, 3, 4], [100, 101, 102, 103, 104]]
        for name, (alloc, off) in {"recv": (0, 0), "y": (0, 4096), "W1": (1, 0), "W3": (1, 8192),
                                   "W2": (1, 16384)}.items():
            row = tables[name]
            assert len(row) == world
            assert row[rank] == (1 << 40) + alloc * (1 << 30) + off  # own buffer by address
            assert row[peer] == (7 << 44 | peer << 36 | alloc << 30) + off
