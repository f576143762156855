"""Star Attention over several GPUs: blocks sharded over the ranks of a process group.

The pages run one host per context block ("Star Attention 完全拆解(一)", Phase 1: every
host gets the anchor block with its own block; "仓库里的真实实现": the host with the last
block appends the query and generated tokens; "通信量:每层每 token 一个标量加一个向量":
each host contributes one (output, log-sum-exp) pair per query token and layer, merged
exactly as in "组装全局结果").  Here a rank owns a contiguous range of blocks of every
sequence.  This module is plumbing only:

* ``block_range`` assigns the ranges (contiguous, sizes differing by at most one);
* ``ShardExchange.gather_merge`` pads a rank's partials to a common count with empty ones
  (O = 0, LSE = -inf, which the merge skips), all-gathers them (outputs and LSEs) on a
  communication stream (NCCL between GPUs; gloo in the CPU tests), and merges every rank's
  partials with the library's ``star_lse_merge`` (or the merge function it is given).

The pages' implementation all-gathers the outputs and the statistics and then waits at a
barrier; here the two gathers run on their own stream so that the next local step can
start, and the merge waits only for its own gathers (no barrier).
"""

from __future__ import annotations

import ctypes
import math
from typing import Callable

import torch
import torch.distributed as dist


def block_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """Blocks [begin, end) of rank `rank` among `world` ranks: contiguous, the first n % world
    ranks one block more.  Every rank needs at least one block (n >= world)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if n < world:
        raise ValueError(f"{n} blocks cannot give each of {world} ranks a block")
    base, extra = divmod(n, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


class ShardExchange:
    """The exchange of one rank: pad, all-gather, merge.

    group: the process group (None = the default one).  device: where the partials live.
    merge_fn(o_all [P, rows, d] f32, lse_all [P, rows] f32) -> (out, lse): defaults to the
    library's star_lse_merge into a bf16 output.
    """

    def __init__(self, n_blocks: int, group=None, device="cuda", merge_fn: Callable | None = None):
        self.group = group
        self.dist = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if self.dist else 1   # one process: no collective
        self.rank = dist.get_rank(group) if self.dist else 0
        self.begin, self.end = block_range(n_blocks, self.world, self.rank)
        self.nmax = math.ceil(n_blocks / self.world)
        self.device = torch.device(device)
        self.merge_fn = merge_fn
        self.use_stream = self.device.type == "cuda"
        self.stream = torch.cuda.Stream(self.device) if self.use_stream else None
        self.nccl = self.dist and dist.get_backend(group) == "nccl"

    @property
    def n_local(self) -> int:
        return self.end - self.begin

    def shard(self):
        from . import StarShard
        return StarShard(self.begin, self.end)

    def _padded(self, o_part: torch.Tensor, lse_part: torch.Tensor, slots: int):
        """The partials padded to `slots` with empty ones (O = 0, LSE = -inf); no copy when
        the rank already has `slots` of them."""
        k, rows, d = o_part.shape
        if k == slots:
            return o_part.to(torch.float32).contiguous(), lse_part.to(torch.float32).contiguous()
        o = torch.zeros((slots, rows, d), dtype=torch.float32, device=o_part.device)
        lse = torch.full((slots, rows), -math.inf, dtype=torch.float32, device=o_part.device)
        o[:k] = o_part
        lse[:k] = lse_part
        return o, lse

    def gather(self, o_part: torch.Tensor, lse_part: torch.Tensor, slots: int | None = None):
        """All ranks' partials: o_part [k, rows, d], lse_part [k, rows] with k <= slots.
        Returns (o_all [world * slots, rows, d], lse_all [world * slots, rows]), rank-major,
        each rank's blocks in order (so they list the context's blocks in order)."""
        slots = self.nmax if slots is None else slots
        if o_part.shape[0] > slots:
            raise ValueError(f"{o_part.shape[0]} partials exceed the {slots} slots per rank")
        if self.use_stream:
            cur = torch.cuda.current_stream(self.device)
            ready = cur.record_event()
            with torch.cuda.stream(self.stream):
                self.stream.wait_event(ready)
                o_send, l_send = self._padded(o_part, lse_part, slots)
                o_all, l_all = self._all_gather(o_send), self._all_gather(l_send)
            cur.wait_event(self.stream.record_event())
            for t in (o_send, l_send, o_all, l_all):
                t.record_stream(cur)  # later uses on the caller's stream keep them alive
        else:
            o_send, l_send = self._padded(o_part, lse_part, slots)
            o_all, l_all = self._all_gather(o_send), self._all_gather(l_send)
        return o_all, l_all

    def _all_gather(self, send: torch.Tensor) -> torch.Tensor:
        """[world * k, ...] from every rank's [k, ...], rank-major."""
        if self.world == 1:
            return send
        recv = torch.empty((self.world * send.shape[0],) + tuple(send.shape[1:]), dtype=send.dtype,
                           device=send.device)
        if self.nccl:
            dist.all_gather_into_tensor(recv, send, group=self.group)
        else:
            dist.all_gather(list(recv.chunk(self.world, 0)), send, group=self.group)
        return recv

    def gather_merge(self, o_part: torch.Tensor, lse_part: torch.Tensor, out=None, lse_out=None,
                     slots: int | None = None):
        """Gather every rank's partials and merge them: the global (O, LSE) of the rows."""
        o_all, lse_all = self.gather(o_part, lse_part, slots)
        if self.merge_fn is not None:
            return self.merge_fn(o_all, lse_all)
        from . import star_lse_merge
        P, rows, d = o_all.shape
        if out is None:
            out = torch.empty((rows, d), dtype=torch.bfloat16, device=o_all.device)
        if lse_out is None:
            lse_out = torch.empty((rows,), dtype=torch.float32, device=o_all.device)
        star_lse_merge(P, rows, d, o_all, lse_all, out.view(rows, d), lse_out.view(rows))
        return out, lse_out


class PeerExchange:
    """One rank's exchange over peer memory (star.h star_exchange): the kernels that finish a
    shard's partials store them straight into every rank's buffer over NVLink, and
    ``star_exchange_merge`` waits for them in this rank's own buffer and merges (no collective
    library on the data path; torch.distributed only carries the buffers' IPC handles once).

    rows, d, slots: the shape of one exchange (rows x d per partial, slots partials per rank).
    Epochs count this exchange's uses, 1, 2, ..., the same on every rank.
    """

    def __init__(self, rows: int, d: int, slots: int, group=None, device="cuda"):
        from . import StarExchange, star_exchange_size, star_ipc_export, star_ipc_open
        self.dist = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if self.dist else 1
        self.rank = dist.get_rank(group) if self.dist else 0
        if self.world > 8:
            raise ValueError("the peer exchange serves up to 8 ranks (one NVLink domain of one node)")
        self.rows, self.d, self.slots = rows, d, slots
        size = star_exchange_size(self.world, slots, rows, d)
        self.buf = torch.zeros(size + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        self.local = self.buf[(-base) % 256:]  # 256-byte aligned start
        ptrs = [0] * self.world
        ptrs[self.rank] = self.local.data_ptr()
        self.opened: list[tuple[int, int]] = []
        if self.world > 1:
            torch.cuda.synchronize(device)  # the zero fill is done before any peer writes
            mine = star_ipc_export(self.local)
            handles = [None] * self.world
            dist.all_gather_object(handles, mine, group=group)
            for w, (h, off) in enumerate(handles):
                if w != self.rank:
                    ptrs[w] = star_ipc_open(h, off)
                    self.opened.append((ptrs[w], off))
            dist.barrier(group=group)  # every buffer is zeroed and mapped before the first push
        self.ex = StarExchange(self.world, self.rank, slots, (ctypes.c_void_p * 8)(*ptrs))
        self.epoch = 0

    def next_epoch(self) -> int:
        self.epoch += 1
        return self.epoch

    def merge(self, out, lse_out=None, epoch: int | None = None):
        from . import star_exchange_merge
        star_exchange_merge(self.ex, self.rows, self.d, self.epoch if epoch is None else epoch, out, lse_out)

    def close(self):
        from . import star_ipc_close
        for ptr, off in self.opened:
            star_ipc_close(ptr, off)
        self.opened = []
