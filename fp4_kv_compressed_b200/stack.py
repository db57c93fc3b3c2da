"""CSA2 layer-stack driver: caches, per-layer buffers and the Full/Reindex/Reuse schedule.

DeepSeek V4.1 Flash study notes, section 2 ("many layers share one global KV"):
every CSA2 layer is statically Full, Reindex or Reuse; the decoder is 1 Full +
4 Reindex + 15 Reuse layers sharing one global KV, each encoder group 1 Full +
5 Reuse.  A Reuse layer takes the most recent selection of its group (nothing
is recomputed); every layer keeps its own query and its own SWA window.  The
decoder order "F U U U X U U U X ..." is this build's reading of the
"Reindex-led groups" of myzaker's CSA2 section.

This module only owns device buffers (allocated through PyTorch) and decides
which library call runs for which layer; every step runs in libcsa2's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _binding as bind

KV_DIM = 512


@dataclass(frozen=True)
class LayerPlan:
    layer: int        # global layer index, execution order
    group: int        # global-KV group
    mode: str         # "F" full, "X" reindex, "U" reuse
    source: int       # layer whose Top-K this layer attends with


def plan_layers(schedules: list[str]) -> list[LayerPlan]:
    """Execution plan of a stack of groups; Reuse points at the nearest preceding
    Full/Reindex layer of its own group.  Raises on a schedule that cannot run
    (a Reindex or Reuse layer with no selection before it)."""
    out: list[LayerPlan] = []
    layer = 0
    for g, sched in enumerate(schedules):
        last_sel = None
        have_pool = False
        for m in sched:
            if m == "F":
                last_sel, have_pool = layer, True
            elif m == "X":
                if not have_pool:
                    raise ValueError(f"group {g}: Reindex layer {layer} before any Full layer")
                last_sel = layer
            elif m == "U":
                if last_sel is None:
                    raise ValueError(f"group {g}: Reuse layer {layer} with nothing to reuse")
            else:
                raise ValueError(f"unknown layer mode {m!r}")
            out.append(LayerPlan(layer, g, m, last_sel))
            layer += 1
    return out


@dataclass(frozen=True)
class GroupSpec:
    ratio: int
    schedule: str
    pool_blocks: int      # 0 = flat indexer
    cap: int              # entries per request


class GlobalKV:
    """Device planes of one global-KV group (FP4 main KV + FP8 indexer K)."""

    def __init__(self, B: int, cap: int, d_idx: int, ratio: int, device):
        self.B, self.cap, self.d_idx, self.ratio = B, cap, d_idx, ratio
        self.codes = torch.zeros(B, cap, KV_DIM // 2, dtype=torch.uint8, device=device)
        self.scales = torch.zeros(B, cap, KV_DIM // 16, dtype=torch.uint8, device=device)
        self.idx_codes = torch.zeros(B, cap, d_idx, dtype=torch.uint8, device=device)
        self.idx_scale = torch.zeros(B, cap, dtype=torch.float32, device=device)
        self.struct = bind.CSA2GlobalKV(self.codes.data_ptr(), self.scales.data_ptr(),
                                        self.idx_codes.data_ptr(), self.idx_scale.data_ptr(),
                                        B, cap, d_idx, ratio)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.codes, self.scales, self.idx_codes, self.idx_scale))


class PagedKV:
    """Device planes of one global-KV group in pages (serving layout): a pool of n_pages
    pages of page_size entries and a block table [B][max_pages] of page ids."""

    def __init__(self, B: int, max_pages: int, page_size: int, n_pages: int, d_idx: int,
                 ratio: int, block_table: torch.Tensor, device):
        if block_table.shape != (B, max_pages) or block_table.dtype != torch.int32:
            raise ValueError("block_table must be int32 [B][max_pages]")
        self.B, self.max_pages, self.page_size, self.n_pages = B, max_pages, page_size, n_pages
        self.d_idx, self.ratio = d_idx, ratio
        rows = n_pages * page_size
        self.codes = torch.zeros(rows, KV_DIM // 2, dtype=torch.uint8, device=device)
        self.scales = torch.zeros(rows, KV_DIM // 16, dtype=torch.uint8, device=device)
        self.idx_codes = torch.zeros(rows, d_idx, dtype=torch.uint8, device=device)
        self.idx_scale = torch.zeros(rows, dtype=torch.float32, device=device)
        self.block_table = block_table.to(device).contiguous()
        self.struct = bind.CSA2PagedKV(self.codes.data_ptr(), self.scales.data_ptr(),
                                       self.idx_codes.data_ptr(), self.idx_scale.data_ptr(),
                                       self.block_table.data_ptr(), B, max_pages, page_size,
                                       n_pages, d_idx, ratio)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.codes, self.scales, self.idx_codes, self.idx_scale, self.block_table))

    def rows_of(self, b: int, n: int) -> torch.Tensor:
        """Pool rows of entries 0..n-1 of request b."""
        e = torch.arange(n, device=self.block_table.device)
        return self.block_table[b][e // self.page_size].long() * self.page_size + e % self.page_size


class SwaRing:
    """One layer's FP8 SWA window ring: token p lives in slot p % window_cap."""

    def __init__(self, B: int, window_cap: int, device):
        self.B, self.window_cap = B, window_cap
        self.codes = torch.zeros(B, window_cap, KV_DIM, dtype=torch.uint8, device=device)
        self.scale = torch.zeros(B, window_cap, dtype=torch.float32, device=device)
        self.struct = bind.CSA2SWA(self.codes.data_ptr(), self.scale.data_ptr(), B, window_cap)


class DecodeStack:
    """All device state of a CSA2 stack for a batch of B requests, Tq queries each."""

    def __init__(self, B: int, H: int, H_I: int, d_idx: int, top_k: int, swa_len: int,
                 groups: list[GroupSpec], Tq: int = 1, window_cap: int | None = None,
                 device="cuda", index_scan: str = "exact", rope=None, page_size: int = 0,
                 page_seed: int = 0):
        if index_scan not in ("exact", "tc"):
            raise ValueError(f"index_scan must be 'exact' or 'tc', not {index_scan!r}")
        if page_size and index_scan != "exact":
            raise ValueError("the paged calls take the exact Full scan")
        # page_size > 0: each group's cache lives in pages of page_size entries (a pool of
        # B * ceil(cap / page_size) pages per group, handed to the requests in a seeded
        # random order through block tables) and every call takes its _paged form
        self.page_size = page_size
        # "exact": the fixed fp32 score order (reproducible Top-K); "tc": the tensor-core
        # scan for prefill chunks (relaxed summation order, see csa2_index_full_tc)
        self.index_scan = index_scan
        # Reuse layers launch with csa2_sparse_attn_decode_reuse and Reindex layers with
        # csa2_index_reindex_settled (overlapping the previous launch); False: the
        # ordinary calls (same results, bit for bit)
        self.reuse_launch = True
        # a _binding.Rope: the main-KV and SWA rows are passed before RoPE and rotated
        # inside the append launches (csa2_quantize_append_rope and the fused attention)
        self.rope = rope
        self.B, self.H, self.H_I, self.d_idx = B, H, H_I, d_idx
        self.top_k, self.swa_len, self.Tq = top_k, swa_len, Tq
        self.groups = groups
        self.device = torch.device(device)
        self.window_cap = window_cap or (swa_len + Tq - 1)
        self.plan = plan_layers([g.schedule for g in groups])
        if page_size:
            self.kv = []
            for i, g in enumerate(groups):
                max_pages = -(-g.cap // page_size)
                perm = torch.randperm(B * max_pages, generator=torch.Generator().manual_seed(page_seed + i))
                self.kv.append(PagedKV(B, max_pages, page_size, B * max_pages, d_idx, g.ratio,
                                       perm.to(torch.int32).view(B, max_pages), device))
        else:
            self.kv = [GlobalKV(B, g.cap, d_idx, g.ratio, device) for g in groups]
        self.swa = [SwaRing(B, self.window_cap, device) for _ in self.plan]
        BT = B * Tq
        dev = self.device
        self.topk = {}
        self.count = {}
        for lp in self.plan:
            if lp.mode in "FX":
                self.topk[lp.layer] = torch.full((B, Tq, top_k), -1, dtype=torch.int32, device=dev)
                self.count[lp.layer] = torch.zeros(B, Tq, dtype=torch.int32, device=dev)
        self.pool = {g: torch.full((B, Tq, max(spec.pool_blocks, 1)), -1, dtype=torch.int32,
                                   device=dev)
                     for g, spec in enumerate(groups)}
        self.out = [torch.zeros(B, Tq, H, KV_DIM, dtype=torch.float32, device=dev)
                    for _ in self.plan]
        self.lse = [torch.zeros(B, Tq, H, dtype=torch.float32, device=dev) for _ in self.plan]
        ws = 256
        for spec in groups:
            ws = max(ws, bind.csa2_workspace_size(bind.CSA2_OP_INDEX_FULL, B, Tq, spec.cap, H,
                                                  top_k, spec.pool_blocks))
            if spec.pool_blocks:
                ws = max(ws, bind.csa2_workspace_size(bind.CSA2_OP_INDEX_REINDEX, B, Tq, 0, H,
                                                      top_k, spec.pool_blocks))
        ws = max(ws, bind.csa2_workspace_size(bind.CSA2_OP_SPARSE_ATTN, B, Tq, 0, H, top_k, 0))
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.softmax_scale = KV_DIM ** -0.5

    def topk_of(self, layer: int) -> torch.Tensor:
        return self.topk[self.plan[layer].source]

    def cache_bytes(self) -> int:
        return sum(g.nbytes() for g in self.kv) + sum(
            r.codes.numel() + r.scale.numel() * 4 for r in self.swa)

    # -----------------------------------------------------------------------------------
    def step(self, *, q_pos, n_max, q, q_idx, w, swa_bf16, swa_start, kv_bf16=None,
             idxk_bf16=None, kv_start=None, stream=None):
        """Run every layer of the stack once, in order.

        q_pos [B][Tq] int32 token positions; n_max[g] >= visible entries of any query of
        group g; q[l] bf16 [B][Tq][H][512]; q_idx[l] bf16 [B][Tq][H_I][d_idx] and w[l]
        fp32 [B][Tq][H_I] for Full/Reindex layers; swa_bf16[l] bf16 [B][T_swa][512] new
        SWA rows at token positions swa_start [B]; kv_bf16[g] / idxk_bf16[g] bf16
        [B][T_kv][...] new entries of group g at entry slots kv_start[g] [B] (None =
        nothing to append).
        """
        first_of_group = {}
        for lp in self.plan:
            first_of_group.setdefault(lp.group, lp.layer)
        T_swa = swa_bf16[0].shape[1] if swa_bf16[0] is not None else 0
        rope = self.rope.struct if self.rope is not None else None

        paged = self.page_size > 0

        def append(*args):
            if paged and args[0] is not None:
                bind.csa2_quantize_append_paged(*args, rope, self.dev_err, stream)
            elif rope is None:
                bind.csa2_quantize_append(*args, self.dev_err, stream)
            else:
                bind.csa2_quantize_append_rope(*args, rope, self.dev_err, stream)

        for lp in self.plan:
            g, l = lp.group, lp.layer
            kv = self.kv[g]
            if l == first_of_group[g] and kv_bf16 is not None and kv_bf16[g] is not None:
                T_kv = kv_bf16[g].shape[1]
                append(kv.struct, kv_bf16[g], idxk_bf16[g], T_kv, kv_start[g], self.swa[l].struct,
                       swa_bf16[l], T_swa, swa_start)
            elif swa_bf16[l] is not None and not self._fuse_swa(T_swa):
                append(None, None, None, 0, None, self.swa[l].struct, swa_bf16[l], T_swa, swa_start)
            spec = self.groups[g]
            if lp.mode == "F":
                full = bind.csa2_index_full_tc if self.index_scan == "tc" else bind.csa2_index_full
                if paged:
                    full = bind.csa2_index_full_paged
                full(kv.struct, q_idx[l], w[l], q_pos, self.Tq, self.H_I, n_max[g],
                     spec.pool_blocks, self.top_k, self.pool[g] if spec.pool_blocks else None,
                     self.topk[l], self.count[l], self.workspace, self.dev_err, stream)
            elif lp.mode == "X":
                # the pool comes from the group's Full layer, whose attention launched in
                # between: the scoring may overlap the previous launch (unless this layer's
                # own SWA append was just launched, which the scoring does not read either)
                if paged:
                    reindex = bind.csa2_index_reindex_paged_settled if self.reuse_launch \
                        else bind.csa2_index_reindex_paged
                else:
                    reindex = bind.csa2_index_reindex_settled if self.reuse_launch else bind.csa2_index_reindex
                reindex(kv.struct, q_idx[l], w[l], q_pos, self.Tq, self.H_I, self.pool[g],
                        spec.pool_blocks, self.top_k, self.topk[l], self.count[l], self.workspace,
                        self.dev_err, stream)
            fused = (l != first_of_group[g] or kv_bf16 is None or kv_bf16[g] is None) \
                and swa_bf16[l] is not None and self._fuse_swa(T_swa)
            if paged:
                attn = bind.csa2_sparse_attn_decode_paged_reuse if fused and lp.mode == "U" and self.reuse_launch \
                    else bind.csa2_sparse_attn_decode_paged
                attn(
                    kv.struct, self.swa[l].struct, swa_bf16[l] if fused else None, q[l], q_pos, self.Tq,
                    self.H, self.topk_of(l), self.top_k, self.swa_len, self.softmax_scale,
                    rope if fused else None, self.out[l], self.lse[l], self.dev_err, stream)
            elif fused and lp.mode == "U" and self.reuse_launch:
                # a Reuse layer: its Top-K and every other input were written two or more
                # launches back (the source layer's attention launched in between), so
                # the launch overlaps the previous one
                bind.csa2_sparse_attn_decode_reuse(
                    kv.struct, self.swa[l].struct, swa_bf16[l], q[l], q_pos, self.Tq, self.H,
                    self.topk_of(l), self.top_k, self.swa_len, self.softmax_scale, rope,
                    self.out[l], self.lse[l], self.dev_err, stream)
            elif fused and rope is not None:
                bind.csa2_sparse_attn_decode_append_rope(
                    kv.struct, self.swa[l].struct, swa_bf16[l], q[l], q_pos, self.Tq, self.H,
                    self.topk_of(l), self.top_k, self.swa_len, self.softmax_scale, rope,
                    self.out[l], self.lse[l], self.workspace, self.dev_err, stream)
            elif fused:     # the layer's SWA row is appended inside the attention launch
                bind.csa2_sparse_attn_decode_append(
                    kv.struct, self.swa[l].struct, swa_bf16[l], q[l], q_pos, self.Tq, self.H,
                    self.topk_of(l), self.top_k, self.swa_len, self.softmax_scale, self.out[l],
                    self.lse[l], self.workspace, self.dev_err, stream)
            else:
                bind.csa2_sparse_attn_decode(kv.struct, self.swa[l].struct, q[l], q_pos, self.Tq,
                                          self.H, self.topk_of(l), self.top_k, self.swa_len,
                                          self.softmax_scale, self.out[l], self.lse[l],
                                          self.workspace, self.dev_err, stream)

    def _fuse_swa(self, T_swa: int) -> bool:
        """Decode (one query token, its own SWA row): the append runs inside the
        attention launch (csa2_sparse_attn_decode_append)."""
        return self.Tq == 1 and T_swa == 1 and self.swa_len > 0

    def launches_per_step(self, append: bool = True) -> int:
        """Kernels one step() launches (with new entries appended)."""
        n = 0
        first = {}
        for lp in self.plan:
            first.setdefault(lp.group, lp.layer)
        for lp in self.plan:
            if lp.layer == first[lp.group] or not self._fuse_swa(self.Tq):
                n += 1                 # quantise-append (the group's entry and/or SWA rows)
            n += {"F": 2, "X": 2, "U": 0}[lp.mode]
            n += 1                     # attention (with the fused SWA append in decode)
        return n

