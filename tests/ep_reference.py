"""Reference restatement of the expert-parallel exchange plan in numpy (test
infrastructure: the library builds the plan on the device with moe_ep_plan;
this is what the tests compare it with, itself checked against a direct
enumeration of the (rank, token, expert) rows in test_ep_plan.py)."""
from dataclasses import dataclass
from typing import List

import numpy as np


@dataclass
class RefPlan:
    send_splits: List[int]
    recv_splits: List[int]
    regroup: np.ndarray         # regrouped row -> received row
    local_offsets: np.ndarray   # [E_loc + 1]
    n_send: int
    n_recv: int


def plan_reference(offsets_all: np.ndarray, rank: int, world: int) -> RefPlan:
    """offsets_all[src] = rank src's [E_r + 1] expert offsets.  Rank r owns
    experts r*E_loc .. (r+1)*E_loc - 1; received rows arrive source by source
    and are regrouped expert by expert, sources ascending."""
    offs = np.asarray(offsets_all, np.int64)
    E_r = offs.shape[1] - 1
    assert E_r % world == 0
    E_loc = E_r // world
    cnt = np.diff(offs, axis=1)
    lo, hi = rank * E_loc, (rank + 1) * E_loc
    send = [int(offs[rank, (r + 1) * E_loc] - offs[rank, r * E_loc]) for r in range(world)]
    mine = cnt[:, lo:hi]
    recv = [int(x) for x in mine.sum(axis=1)]
    local_offsets = np.concatenate([[0], np.cumsum(mine.sum(axis=0))]).astype(np.int32)
    src_base = np.concatenate([[0], np.cumsum(recv)])[:-1]
    regroup = np.empty(int(mine.sum()), np.int32)
    for e in range(E_loc):
        at = local_offsets[e]
        for src in range(world):
            n = int(mine[src, e])
            first = src_base[src] + int(mine[src, :e].sum())
            regroup[at:at + n] = np.arange(first, first + n)
            at += n
    return RefPlan(send, recv, regroup, local_offsets, int(sum(send)), int(sum(recv)))
