"""How one LSA layer or decode batch is divided between the ranks of a
job (one process per GPU).

The path partitions without a collective on its data path:
* by kv-head: each rank owns hkv / N kv-heads with the hq / N query heads
  of their GQA groups (their K/V, bucket cache and tree); a head's index
  lists and outputs depend only on that head's keys and its group's queries
  (essay "《卡片柜》" ch. 3: every kv-head keeps its own bucket cache);
* by request in decode: each rank owns a contiguous slice of the batch.
"""
from __future__ import annotations


def head_range(hkv: int, hq: int, world: int, rank: int):
    """(h0, h1, q0, q1): the kv-heads [h0, h1) and query heads [q0, q1) of
    `rank` when hkv kv-heads are split evenly over `world` ranks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    if hkv % world or hq % hkv:
        raise ValueError(f"{hkv} kv-heads do not split evenly over {world} ranks")
    per = hkv // world
    G = hq // hkv
    return rank * per, (rank + 1) * per, rank * per * G, (rank + 1) * per * G


def request_range(batch: int, world: int, rank: int):
    """(r0, r1): the decode requests of `rank` (contiguous, sizes differing
    by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    return rank * batch // world, (rank + 1) * batch // world
