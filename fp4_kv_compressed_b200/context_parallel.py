"""Context parallel: one long request's global KV split by entry range across ranks.

DeepSeek V4.1 Flash study notes, section 2 (report Figure 5): the Full-layer scan is
the only per-query cost that grows with the context, so a single request too long for
one GPU is split into contiguous slices of its global-KV entries, one per rank.  Per
Full layer and decode step:

1. every rank scans its slice: ``csa2_index_full_slice`` -> its local pool and Top-K
   as candidate keys (order key << 32 | ~global id);
2. the candidate keys are all-gathered (rank order = ascending slice order);
3. every rank merges them: ``csa2_index_merge`` -> the global pool / Top-K (exact:
   every item of a global selection is in its own slice's local selection) and the
   part that falls in its own slice, as slice-local ids;
4. every rank attends over its part (the rank holding the query's window also over
   the window), the partial (o, lse) are all-gathered and ``csa2_attn_combine`` forms
   the one softmax over the union.

The only exchanges are the two all-gathers; both move small tensors (pool_blocks +
top_k keys of 8 bytes, then H x 512 fp32 + H lse per query).  Every step runs in the
library's kernels; this module only allocates buffers, orders the calls and does the
collectives through ``torch.distributed`` (NCCL on GPUs).  The compute calls go
through a ``backend`` object (the C library by default) and the gather through a
``gather`` callable, so that the host logic can be exercised without a GPU.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _binding as bind

ALIGN = 64          # slice bounds are multiples of 64 entries (whole 8- and 64-blocks)


def slice_bounds(n_entries: int, world: int, align: int = ALIGN) -> list[tuple[int, int]]:
    """Contiguous slices [lo, hi) of n_entries entries over `world` ranks; every lo is a
    multiple of `align`, the last slice ends at n_entries (some slices may be empty)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    per = -(-n_entries // world)
    per = -(-per // align) * align
    out = []
    for r in range(world):
        lo = min(n_entries, r * per)
        hi = min(n_entries, lo + per) if r < world - 1 else n_entries
        out.append((lo, max(lo, hi)))
    return out


def dist_gather(t: torch.Tensor) -> torch.Tensor:
    """All-gather of a tensor over the default process group: [world, *t.shape]."""
    import torch.distributed as dist
    world = dist.get_world_size()
    t = t.contiguous()
    out = torch.empty((world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(out, t)       # concatenation along dim 0, rank order
    return out.view((world,) + tuple(t.shape))


class LibraryBackend:
    """The C library's calls (device tensors)."""

    @staticmethod
    def index_full_slice(kv, entry_lo, q_idx, w, q_pos, Tq, H_I, n_max, pool_blocks, top_k,
                         pool_keys, topk_keys, workspace, dev_err, stream):
        bind.csa2_index_full_slice(kv.struct, entry_lo, q_idx, w, q_pos, Tq, H_I, n_max,
                                   pool_blocks, top_k, pool_keys if pool_blocks else None,
                                   topk_keys, workspace, dev_err, stream)

    @staticmethod
    def index_merge(lists, BT, n_lists, list_len, k, lo, hi, ids_out, count_out, local_out,
                    stream):
        bind.csa2_index_merge(lists, BT, n_lists, list_len, k, lo, hi, ids_out, count_out,
                              local_out, stream)

    @staticmethod
    def attention(kv, swa, q, q_pos, Tq, H, topk_local, top_k, swa_len, scale, out, lse,
                  dev_err, stream):
        bind.csa2_sparse_attn_decode(kv.struct, swa.struct if swa is not None else None, q,
                                     q_pos, Tq, H, topk_local, top_k, swa_len, scale, out, lse,
                                     None, dev_err, stream)

    @staticmethod
    def combine(o_parts, lse_parts, n_parts, rows, out, lse_out, stream):
        bind.csa2_attn_combine(o_parts, lse_parts, n_parts, rows, out, lse_out, stream)


@dataclass
class FullResult:
    pool: torch.Tensor | None         # [B][Tq][pool_blocks] global block ids (-1 padded)
    pool_local: torch.Tensor | None   # the blocks of this rank's slice, as slice-local blocks
    topk: torch.Tensor                # [B][Tq][top_k] global entry ids (-1 padded)
    topk_local: torch.Tensor          # this rank's part, as slice-local entry ids (-1 elsewhere)
    count: torch.Tensor               # [B][Tq]


class ContextShard:
    """One rank's slice [lo, hi) of the global-KV entries of a batch of requests.

    `kv` is a GlobalKV whose cap covers the slice (entry e of it is global entry lo + e);
    `window` tells whether this rank holds the layers' SWA rings (the newest tokens)."""

    def __init__(self, kv, lo: int, hi: int, rank: int, world: int, window: bool,
                 gather=dist_gather, backend=LibraryBackend):
        if lo % ALIGN:
            raise ValueError(f"slice start {lo} is not a multiple of {ALIGN}")
        self.kv, self.lo, self.hi, self.rank, self.world = kv, lo, hi, rank, world
        self.window = window
        self.gather, self.backend = gather, backend

    def local_n_max(self, q_pos: torch.Tensor) -> int:
        """The largest number of this slice's entries any query sees."""
        t = int(q_pos.max().item())
        n_vis = (t + 1) // self.kv.ratio
        return max(0, min(self.hi, n_vis) - self.lo)

    def scan(self, q_idx, w, q_pos, Tq: int, H_I: int, pool_blocks: int, top_k: int,
             workspace, n_max: int | None = None, dev_err=None, stream=None):
        """Step 1: this slice's local selections as candidate keys
        (pool_keys [B][Tq][pool_blocks] or None, topk_keys [B][Tq][top_k], int64)."""
        B = q_pos.shape[0]
        dev = q_pos.device
        n_max = self.local_n_max(q_pos) if n_max is None else n_max
        pool_keys = (torch.zeros(B, Tq, pool_blocks, dtype=torch.int64, device=dev)
                     if pool_blocks else None)
        topk_keys = torch.zeros(B, Tq, top_k, dtype=torch.int64, device=dev)
        if n_max > 0:
            self.backend.index_full_slice(self.kv, self.lo, q_idx, w, q_pos, Tq, H_I, n_max,
                                          pool_blocks, top_k, pool_keys, topk_keys, workspace,
                                          dev_err, stream)
        return pool_keys, topk_keys

    def merge(self, pool_lists, topk_lists, stream=None) -> FullResult:
        """Step 3: the global selections from every slice's candidate keys, gathered
        shard-major ([world][B][Tq][n])."""
        world, B, Tq, K = topk_lists.shape
        dev = topk_lists.device
        BT = B * Tq
        res_pool = res_pool_local = None
        if pool_lists is not None:
            P = pool_lists.shape[-1]
            res_pool = torch.empty(B, Tq, P, dtype=torch.int32, device=dev)
            res_pool_local = torch.empty_like(res_pool)
            self.backend.index_merge(pool_lists, BT, world, P, P, self.lo // 8, -(-self.hi // 8),
                                     res_pool, None, res_pool_local, stream)
        topk = torch.empty(B, Tq, K, dtype=torch.int32, device=dev)
        topk_local = torch.empty_like(topk)
        count = torch.empty(B, Tq, dtype=torch.int32, device=dev)
        self.backend.index_merge(topk_lists, BT, world, K, K, self.lo, self.hi, topk, count,
                                 topk_local, stream)
        return FullResult(res_pool, res_pool_local, topk, topk_local, count)

    def full_select(self, q_idx, w, q_pos, Tq: int, H_I: int, pool_blocks: int, top_k: int,
                    workspace, n_max: int | None = None, dev_err=None,
                    stream=None) -> FullResult:
        """Steps 1-3: the Full layer over the whole (split) context."""
        pool_keys, topk_keys = self.scan(q_idx, w, q_pos, Tq, H_I, pool_blocks, top_k,
                                         workspace, n_max, dev_err, stream)
        pool_lists = self.gather(pool_keys) if pool_keys is not None else None
        return self.merge(pool_lists, self.gather(topk_keys), stream)

    def attend_partial(self, swa, q, q_pos, Tq: int, H: int, topk_local, top_k: int,
                       swa_len: int, scale: float, dev_err=None, stream=None):
        """Step 4a: this rank's normalised partial attention (o, lse)."""
        B = q.shape[0]
        dev = q.device
        o = torch.zeros(B, Tq, H, 512, dtype=torch.float32, device=dev)
        l = torch.full((B, Tq, H), float("-inf"), dtype=torch.float32, device=dev)
        self.backend.attention(self.kv, swa if self.window else None, q, q_pos, Tq, H, topk_local,
                               top_k, swa_len if self.window else 0, scale, o, l, dev_err, stream)
        return o, l

    def combine(self, o_parts, l_parts, stream=None):
        """Step 4b: one softmax from the gathered partials ([world][B][Tq][H][512] and
        [world][B][Tq][H])."""
        world = o_parts.shape[0]
        out = torch.empty(o_parts.shape[1:], dtype=torch.float32, device=o_parts.device)
        lse = torch.empty(l_parts.shape[1:], dtype=torch.float32, device=l_parts.device)
        self.backend.combine(o_parts, l_parts, world, l_parts[0].numel(), out, lse, stream)
        return out, lse

    def attend(self, swa, q, q_pos, Tq: int, H: int, topk_local, top_k: int, swa_len: int,
               scale: float, dev_err=None, stream=None):
        """Step 4: partial attention, all-gather, combine.  Returns (out [B][Tq][H][512],
        lse [B][Tq][H]) of the softmax over the whole selection and window."""
        o, l = self.attend_partial(swa, q, q_pos, Tq, H, topk_local, top_k, swa_len, scale,
                                   dev_err, stream)
        return self.combine(self.gather(o), self.gather(l), stream)
