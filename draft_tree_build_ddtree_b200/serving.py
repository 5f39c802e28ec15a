"""Continuous DDTree rounds over a request batch sharded across GPUs.

One process per GPU.  Requests are independent, so a batch shards by
request with no collective on the data path: request r lives on rank
r mod world, with its KV pages, and each rank runs ``ddtree_round`` over its
own shard.  After a round each request's next round starts from what the
round committed ("DDTree Deep Dive" §5 and §6: the accepted path is
compacted into the cache, the prefix grows by accept_len, and the target's
token at the last accepted node is the next root):

    prefix_len <- new_prefix_len,   root_token <- next_bonus

Both hand-overs are pointer swaps between two buffers (the round writes
one and reads the other), so a loop step is one ``ddtree_round`` call.  The
only collective is an all-gather of every request's (accept_len,
next_bonus, new_prefix_len) into request order, for the scheduler.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch

from . import RoundBuffers, ddtree_round


def shard_of(n_req: int, world: int, rank: int) -> List[int]:
    """The requests rank ``rank`` owns: r with r mod world == rank, ascending."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return list(range(rank, n_req, world))


def gather_by_request(local: torch.Tensor, n_req: int, world: int, rank: int) -> torch.Tensor:
    """All-gather each rank's per-request rows into request order.

    ``local`` is [len(shard_of(n_req, world, rank)), m] (any device the
    process group's backend takes); returns [n_req, m] on the same device.
    With world == 1 it is the identity, with no collective.
    """
    if world == 1:
        return local
    per = math.ceil(n_req / world)
    m = local.shape[1]
    pad = torch.zeros((per, m), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    torch.distributed.all_gather(parts, pad)
    out = torch.empty((n_req, m), dtype=local.dtype, device=local.device)
    for q in range(world):
        idx = shard_of(n_req, world, q)
        out[idx] = parts[q][:len(idx)]
    return out


@dataclasses.dataclass
class ServingLoop:
    """Continuous rounds over one rank's shard.

    ``rb`` holds the shard's buffers (its requests only).  Two RoundArgs
    alternate the roles of (prefix_len, new_prefix_len) and (root_token,
    next_bonus), so round k + 1 reads what round k wrote.
    """
    rb: RoundBuffers
    requests: List[int]
    n_total: int
    world: int = 1
    rank: int = 0
    rounds: int = 0

    def __post_init__(self):
        rb = self.rb
        self._bufs = [(rb.prefix_len, rb.root_token),
                      (torch.empty_like(rb.prefix_len), torch.empty_like(rb.root_token))]
        self._args = []
        for k in range(2):
            (p_in, r_in), (p_out, r_out) = self._bufs[k], self._bufs[1 - k]
            rb.prefix_len, rb.root_token = p_in, r_in
            rb.acc.new_prefix_len, rb.acc.next_bonus = p_out, r_out
            self._args.append(rb.args())
        self._select(0)

    def _select(self, k: int):
        rb = self.rb
        (p_in, r_in), (p_out, r_out) = self._bufs[k], self._bufs[1 - k]
        rb.prefix_len, rb.root_token = p_in, r_in
        rb.acc.new_prefix_len, rb.acc.next_bonus = p_out, r_out
        rb._args = self._args[k]

    @property
    def args(self):
        """The RoundArgs the next step launches with."""
        return self._args[self.rounds % 2]

    def step(self, gather: bool = True) -> Optional[torch.Tensor]:
        """One round on the current stream; returns [n_total, 3] int32
        (accept_len, next_bonus, new_prefix_len) in request order when
        ``gather``."""
        k = self.rounds % 2
        self._select(k)
        ddtree_round(self.rb, self._args[k])
        self.rounds += 1
        if not gather:
            return None
        rb = self.rb
        local = torch.stack([rb.acc.accept_len, rb.acc.next_bonus, rb.acc.new_prefix_len], dim=1)
        return gather_by_request(local, self.n_total, self.world, self.rank)

    def committed(self):
        """(prefix_len, root_token) the next round starts from."""
        p, r = self._bufs[self.rounds % 2]
        return p, r
