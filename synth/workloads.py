"""The five synthetic CSA2 workloads and per-request input regeneration.

Shapes follow the DeepSeek V4.1 Flash pages as fixed for this build:
512-channel shared K=V latent entries, 128-token per-layer SWA window,
Top-512 out of a pool of 2048 blocks x 8 positions (decoder) or a flat
Top-512 (encoder groups, 2 tokens per entry).  Inputs are drawn by the
counter-based generator in :mod:`synth`, so any request of any workload can be
regenerated alone, on the host, with the bits the GPU harness used.

Nothing here quantises, scores, selects or attends.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

from . import POS_STRIDE, Q_STRIDE, row_indices, rows_normal_bf16, rows_uniform_f32, \
    hash_u32, tensor_keys, normal_bf16

KV_DIM = 512            # shared K=V latent width
DECODER_SCHEDULE = "FUUUXUUUXUUUXUUUXUUU"   # 1 Full + 4 Reindex + 15 Reuse
ENCODER_SCHEDULE = "FUUUUU"                 # 1 Full + 5 Reuse, flat indexer
# RoPE runs (pre-RoPE rows rotated inside the append): the last 64 of the 512 latent
# channels.  The pages give neither the rotated channels nor the angles; the angles
# come from synth.rope_table.
ROPE_START, ROPE_PAIRS = 448, 32


@dataclass(frozen=True)
class Group:
    """One global-KV group: its compression ratio, layer modes and indexer kind."""
    ratio: int
    schedule: str
    pool_blocks: int          # 0 = flat Top-K over all visible entries


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    ctx: int                  # tokens visible to the (last) query, current token included
    H: int
    H_I: int
    d_I: int
    top_k: int
    swa_len: int
    groups: tuple
    Tq: int = 1               # query tokens per request (prefill chunk when > 1)
    chan_scale: bool = False  # per-channel log-uniform [0.25, 4] scale on main KV and SWA
    planted: int = 0          # planted high-score index positions per request
    description: str = ""
    b0: int = 0               # global index of request 0 (ranks hold disjoint requests)

    # ---- derived shapes -------------------------------------------------------------------
    @property
    def first_q_pos(self) -> int:
        return self.ctx - self.Tq

    def q_positions(self) -> list[int]:
        return [self.first_q_pos + i for i in range(self.Tq)]

    def entries(self, g: int) -> int:
        """Entries held by group g once every query token has been appended."""
        return self.ctx // self.groups[g].ratio

    def cap(self, g: int) -> int:
        return self.entries(g)

    @property
    def window_cap(self) -> int:
        return self.swa_len + self.Tq - 1

    @property
    def layers(self) -> list[tuple[int, str]]:
        """(group, mode) of every CSA2 layer in execution order."""
        out = []
        for g, grp in enumerate(self.groups):
            for m in grp.schedule:
                out.append((g, m))
        return out

    # ---- generator streams ----------------------------------------------------------------
    def _scale(self, device) -> torch.Tensor | None:
        if not self.chan_scale:
            return None
        # one draw per channel, log-uniform in [0.25, 4]; computed in fp64 on the host.
        idx = torch.arange(KV_DIM, dtype=torch.int64)
        h = hash_u32(idx, tensor_keys(self.seed, "chan_scale"))
        u = (h.double() + 0.5) / 2.0 ** 32
        s = torch.pow(2.0, 4.0 * u - 2.0).to(torch.float32)
        return s.to(device)

    def _apply_scale(self, x: torch.Tensor) -> torch.Tensor:
        s = self._scale(x.device)
        if s is None:
            return x
        return (x.float() * s).to(torch.bfloat16)

    def main_kv(self, g: int, b: int, start: int, count: int, device="cpu") -> torch.Tensor:
        """bf16 [count][512] post-RoPE main KV entries of group g, request b."""
        x = rows_normal_bf16(self.seed, f"g{g}.kv", self.b0 + b, start, count, KV_DIM, device)
        return self._apply_scale(x)

    def idx_k(self, g: int, b: int, start: int, count: int, device="cpu") -> torch.Tensor:
        """bf16 [count][d_I] indexer-K rows of group g, request b (planted rows included)."""
        x = rows_normal_bf16(self.seed, f"g{g}.idxk", self.b0 + b, start, count, self.d_I,
                             device)
        if self.planted and g == self.decoder_group:
            pos, rows = self.planted_rows(b)
            for p, r in zip(pos, rows):
                if start <= p < start + count:
                    x[p - start] = r.to(device)
        return x

    def swa(self, layer: int, b: int, start: int, count: int, device="cpu") -> torch.Tensor:
        """bf16 [count][512] SWA rows of one layer for token positions [start, start+count)."""
        x = rows_normal_bf16(self.seed, f"L{layer}.swa", self.b0 + b, start, count, KV_DIM,
                             device)
        return self._apply_scale(x)

    def q(self, layer: int, b: int, device="cpu") -> torch.Tensor:
        """bf16 [Tq][H][512] attention queries of one layer."""
        x = rows_normal_bf16(self.seed, f"L{layer}.q", self.b0 + b, 0, self.Tq * self.H, KV_DIM,
                             device, stride=Q_STRIDE)
        return x.view(self.Tq, self.H, KV_DIM)

    def q_idx(self, layer: int, b: int, device="cpu") -> torch.Tensor:
        """bf16 [Tq][H_I][d_I] index queries of one layer."""
        x = rows_normal_bf16(self.seed, f"L{layer}.qidx", self.b0 + b, 0, self.Tq * self.H_I,
                             self.d_I, device, stride=Q_STRIDE)
        return x.view(self.Tq, self.H_I, self.d_I)

    def w(self, layer: int, b: int, device="cpu") -> torch.Tensor:
        """fp32 [Tq][H_I] index-head weights, U(0,1)."""
        x = rows_uniform_f32(self.seed, f"L{layer}.w", self.b0 + b, 0, self.Tq, self.H_I, device)
        return x.view(self.Tq, self.H_I)

    # ---- structure ------------------------------------------------------------------------
    @property
    def decoder_group(self) -> int:
        return len(self.groups) - 1

    @property
    def decoder_full_layer(self) -> int:
        base = sum(len(g.schedule) for g in self.groups[:-1])
        return base + self.groups[-1].schedule.index("F")

    def planted_rows(self, b: int):
        """Planted positions of request b and their bf16 index-K rows.

        Positions are distinct, drawn in [0, N - 128) of the decoder group; each
        row is 4 * sign(sum_h w_h q_h) over the decoder Full layer's index query,
        evaluated in fp64 on the host.
        """
        n = self.entries(self.decoder_group) - 128
        if self.planted == 0 or n <= 0:
            return [], []
        keys = tensor_keys(self.seed, "planted")
        pos: list[int] = []
        j = 0
        while len(pos) < self.planted:
            h = int(hash_u32(torch.tensor([(self.b0 + b) * 4096 + j], dtype=torch.int64),
                             keys)[0])
            p = h % n
            if p not in pos:
                pos.append(p)
            j += 1
        L = self.decoder_full_layer
        qi = self.q_idx(L, b).double()[0]          # [H_I][d_I]
        wv = self.w(L, b).double()[0]              # [H_I]
        direction = (wv[:, None] * qi).sum(0)      # [d_I]
        row = (4.0 * torch.sign(direction)).to(torch.bfloat16)
        return pos, [row.clone() for _ in pos]


def _dec(B, ctx, H, H_I, d_I, top_k, pool, seed, **kw):
    return Workload(groups=(Group(1, DECODER_SCHEDULE, pool),), B=B, ctx=ctx, H=H, H_I=H_I,
                    d_I=d_I, top_k=top_k, swa_len=128, seed=seed, **kw)


WORKLOADS = {
    "tiny_full_layer": Workload(
        name="tiny_full_layer", seed=1001, B=1, ctx=4096, H=16, H_I=4, d_I=64, top_k=64,
        swa_len=128, groups=(Group(1, "F", 64),),
        description="1 request, context 4096, 16 heads, 4x64 index heads, Top-64, pool 64x8"),
    "decoder_group_32k": _dec(
        8, 32768, 64, 4, 128, 512, 2048, 1002, name="decoder_group_32k", planted=8,
        description="batch 8, context 32768, decoder group F+4X+15U, 8 planted positions"),
    "prefill_chunk_enc": Workload(
        name="prefill_chunk_enc", seed=1003, B=1, ctx=65536 + 2048, H=64, H_I=4, d_I=128,
        top_k=512, swa_len=128, Tq=2048, groups=(Group(2, ENCODER_SCHEDULE, 0),),
        description="2048 causal query tokens after a 65536-token prefix, ratio 2, F+5U flat"),
    "decode_128k": _dec(
        64, 131072, 64, 4, 128, 512, 2048, 1004, name="decode_128k", chan_scale=True,
        description="batch 64, context 131072, decoder stack F+4X+15U, per-channel scales"),
    "decode_1m": Workload(
        name="decode_1m", seed=1005, B=4, ctx=1 << 20, H=64, H_I=4, d_I=128, top_k=512,
        swa_len=128,
        groups=(Group(2, ENCODER_SCHEDULE, 0), Group(2, ENCODER_SCHEDULE, 0),
                Group(2, ENCODER_SCHEDULE, 0), Group(1, DECODER_SCHEDULE, 2048)),
        description="batch 4, context 1M, 3 encoder groups (ratio 2, flat) + decoder group"),
}


def small_variant(w: Workload, *, B=None, ctx=None, H=None, Tq=None, name=None,
                  b0=None) -> Workload:
    """A reduced copy of a workload (same structure and seeds) for oracle-sized tests;
    b0 selects which global requests the copy holds."""
    d = dict(w.__dict__)
    if b0 is not None:
        d["b0"] = b0
    if B is not None:
        d["B"] = B
    if ctx is not None:
        d["ctx"] = ctx
    if H is not None:
        d["H"] = H
    if Tq is not None:
        d["Tq"] = Tq
    d["name"] = name or (w.name + "_small")
    return Workload(**d)


# ---- batched row generation (all requests at once, same bits as the per-request calls) ----
def batch_rows_normal_bf16(seed: int, name: str, B: int, start: int, count: int, width: int,
                           device="cpu", stride: int = POS_STRIDE, b0: int = 0) -> torch.Tensor:
    """[B][count][width] bf16; row (b, start+i) equals rows_normal_bf16(..., b0 + b, start,
    ...)[i]."""
    b = (b0 + torch.arange(B, dtype=torch.int64, device=device)).view(B, 1, 1)
    p = (start + torch.arange(count, dtype=torch.int64, device=device)).view(1, count, 1)
    c = torch.arange(width, dtype=torch.int64, device=device).view(1, 1, width)
    idx = (b * stride + p) * width + c
    return normal_bf16(seed, name, idx)


def _main_kv_batch(self: Workload, g: int, start: int, count: int, device="cpu"):
    x = batch_rows_normal_bf16(self.seed, f"g{g}.kv", self.B, start, count, KV_DIM, device,
                               b0=self.b0)
    return self._apply_scale(x)


def _idx_k_batch(self: Workload, g: int, start: int, count: int, device="cpu"):
    x = batch_rows_normal_bf16(self.seed, f"g{g}.idxk", self.B, start, count, self.d_I, device,
                               b0=self.b0)
    if self.planted and g == self.decoder_group:
        for b in range(self.B):
            pos, rows = self.planted_rows(b)
            for p, r in zip(pos, rows):
                if start <= p < start + count:
                    x[b, p - start] = r.to(device)
    return x


def _swa_batch(self: Workload, layer: int, start: int, count: int, device="cpu"):
    x = batch_rows_normal_bf16(self.seed, f"L{layer}.swa", self.B, start, count, KV_DIM, device,
                               b0=self.b0)
    return self._apply_scale(x)


def _q_batch(self: Workload, layer: int, device="cpu"):
    x = batch_rows_normal_bf16(self.seed, f"L{layer}.q", self.B, 0, self.Tq * self.H, KV_DIM,
                               device, stride=Q_STRIDE, b0=self.b0)
    return x.view(self.B, self.Tq, self.H, KV_DIM)


def _q_idx_batch(self: Workload, layer: int, device="cpu"):
    x = batch_rows_normal_bf16(self.seed, f"L{layer}.qidx", self.B, 0, self.Tq * self.H_I,
                               self.d_I, device, stride=Q_STRIDE, b0=self.b0)
    return x.view(self.B, self.Tq, self.H_I, self.d_I)


def _w_batch(self: Workload, layer: int, device="cpu"):
    from . import uniform_f32
    b = (self.b0 + torch.arange(self.B, dtype=torch.int64, device=device)).view(self.B, 1, 1)
    r = torch.arange(self.Tq, dtype=torch.int64, device=device).view(1, self.Tq, 1)
    c = torch.arange(self.H_I, dtype=torch.int64, device=device).view(1, 1, self.H_I)
    idx = (b * Q_STRIDE + r) * self.H_I + c
    return uniform_f32(self.seed, f"L{layer}.w", idx)


Workload.main_kv_batch = _main_kv_batch
Workload.idx_k_batch = _idx_k_batch
Workload.swa_batch = _swa_batch
Workload.q_batch = _q_batch
Workload.q_idx_batch = _q_idx_batch
Workload.w_batch = _w_batch
