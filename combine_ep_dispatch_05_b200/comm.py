"""Connecting the ranks of a communicator (include/ep_comm.h) over
torch.distributed: every rank's connection record goes to every rank, in rank
order (an all-gather of objects), and each rank then maps the others' memory.
The EP_SYNC_HOST barrier is the process group's barrier."""
from __future__ import annotations

from . import binding as b


def gather_records(record: bytes, dist, group=None) -> list:
    """All ranks' connection records, in rank order."""
    recs = [None] * dist.get_world_size(group)
    dist.all_gather_object(recs, record, group=group)
    return recs


def create_and_connect(cfg, dist, sync: int = b.EP_SYNC_DEVICE, group=None) -> int:
    """Create this rank's communicator (rank = the process group's rank) and
    connect it to every other rank's. Collective: every rank calls it."""
    rank = dist.get_rank(group)
    barrier = (lambda: dist.barrier(group=group)) if sync == b.EP_SYNC_HOST else None
    comm = b.ep_comm_create(cfg, rank, sync, barrier=barrier)
    try:
        b.ep_comm_connect(comm, gather_records(b.ep_comm_handle(comm), dist, group))
    except BaseException:
        b.ep_comm_destroy(comm)
        raise
    return comm
