"""Device harness for the synthetic CSA2 workloads (tests and benchmark).

Builds a workload's caches on the GPU through the library's public API
(csa2_quantize_append on bf16 rows drawn by the seeded generator, chunk by
chunk), and prepares the device inputs of one step: the current token's new
entries and SWA rows, each layer's queries, and the positions.  A step re-runs
the same token each time (appending it overwrites the same slots), so every
timed step does identical work.

Layout of a step for query tokens t0 .. t0+Tq-1:
  * before the step, group g holds entries 0 .. t0 // ratio - 1 and each layer's
    ring holds tokens t0 - swa_len + 1 .. t0 - 1;
  * the step appends entries t0 // ratio .. ctx // ratio - 1 and SWA tokens
    t0 .. t0 + Tq - 1, then runs every layer in order.
"""
from __future__ import annotations

import torch

import synth
from fp4_kv_compressed_b200 import (DecodeStack, GroupSpec, Rope, csa2_quantize_append,
                                    csa2_quantize_append_paged, csa2_quantize_append_rope)
from synth.workloads import ROPE_PAIRS, ROPE_START, Workload


class DeviceWorkload:
    def __init__(self, wl: Workload, device="cuda", chunk_elems: int = 1 << 25, fill=True,
                 index_scan: str = "exact", rope: bool = False, page_size: int = 0):
        self.wl = wl
        self.device = torch.device(device)
        self.rope = (Rope(synth.rope_table(wl.ctx, ROPE_PAIRS), ROPE_START, ROPE_PAIRS, device)
                     if rope else None)
        self.groups = [GroupSpec(g.ratio, g.schedule, g.pool_blocks, wl.entries(i))
                       for i, g in enumerate(wl.groups)]
        self.stack = DecodeStack(wl.B, wl.H, wl.H_I, wl.d_I, wl.top_k, wl.swa_len, self.groups,
                                 Tq=wl.Tq, window_cap=wl.window_cap, device=device,
                                 index_scan=index_scan, rope=self.rope, page_size=page_size)
        self.t0 = wl.first_q_pos
        self.chunk_elems = chunk_elems
        if fill:
            self.fill_caches()
        self.inputs = self.step_inputs()

    # ---------------------------------------------------------------------------------------
    def fill_caches(self):
        wl, dev, st = self.wl, self.device, self.stack
        for g, spec in enumerate(self.groups):
            n_before = self.t0 // spec.ratio
            chunk = max(1, self.chunk_elems // (wl.B * 512))
            for s in range(0, n_before, chunk):
                c = min(chunk, n_before - s)
                kv = wl.main_kv_batch(g, s, c, dev).contiguous()
                ik = wl.idx_k_batch(g, s, c, dev).contiguous()
                start = torch.full((wl.B,), s, dtype=torch.int32, device=dev)
                self._append(st.kv[g].struct, kv, ik, c, start, None, None, 0, None)
        p0 = max(0, self.t0 - (wl.swa_len - 1))
        cnt = self.t0 - p0
        if cnt > 0:
            start = torch.full((wl.B,), p0, dtype=torch.int32, device=dev)
            for lp in st.plan:
                rows = wl.swa_batch(lp.layer, p0, cnt, dev).contiguous()
                self._append(None, None, None, 0, None, st.swa[lp.layer].struct, rows, cnt, start)
        torch.cuda.synchronize(dev)

    def _append(self, *args):
        if self.stack.page_size and args[0] is not None:
            csa2_quantize_append_paged(*args, self.rope.struct if self.rope is not None else None,
                                       self.stack.dev_err)
        elif self.rope is None:
            csa2_quantize_append(*args, self.stack.dev_err)
        else:
            csa2_quantize_append_rope(*args, self.rope.struct, self.stack.dev_err)

    def step_inputs(self, device=None) -> dict:
        wl = self.wl
        dev = torch.device(device) if device is not None else self.device
        st = self.stack
        kv_bf16, idxk_bf16, kv_start, n_max = [], [], [], []
        for g, spec in enumerate(self.groups):
            e0 = self.t0 // spec.ratio
            n = wl.entries(g)
            n_max.append(n)
            if n > e0:
                kv_bf16.append(wl.main_kv_batch(g, e0, n - e0, dev).contiguous())
                idxk_bf16.append(wl.idx_k_batch(g, e0, n - e0, dev).contiguous())
            else:
                kv_bf16.append(None)
                idxk_bf16.append(None)
            kv_start.append(torch.full((wl.B,), e0, dtype=torch.int32, device=dev))
        q, q_idx, w, swa = [], [], [], []
        for lp in st.plan:
            q.append(wl.q_batch(lp.layer, dev).contiguous())
            if lp.mode in "FX":
                q_idx.append(wl.q_idx_batch(lp.layer, dev).contiguous())
                w.append(wl.w_batch(lp.layer, dev).contiguous())
            else:
                q_idx.append(None)
                w.append(None)
            swa.append(wl.swa_batch(lp.layer, self.t0, wl.Tq, dev).contiguous())
        q_pos = (self.t0 + torch.arange(wl.Tq, dtype=torch.int32, device=dev)).repeat(wl.B, 1)
        return dict(q_pos=q_pos.contiguous(), n_max=n_max, q=q, q_idx=q_idx, w=w, swa_bf16=swa,
                    swa_start=torch.full((wl.B,), self.t0, dtype=torch.int32, device=dev),
                    kv_bf16=kv_bf16, idxk_bf16=idxk_bf16, kv_start=kv_start)

    def step(self, inputs: dict | None = None, stream=None):
        self.stack.step(**(inputs or self.inputs), stream=stream)

    # ---------------------------------------------------------------------------------------
    def request_state(self, b: int) -> dict:
        """Host copies of request b's caches and every layer's outputs (after a step);
        contiguous caches only."""
        if self.stack.page_size:
            raise ValueError("request_state reads the contiguous cache layout")
        st = self.stack
        out = {"kv": [], "swa": [], "topk": {}, "count": {}, "pool": {}, "out": [], "lse": []}
        for g in st.kv:
            out["kv"].append(dict(codes=g.codes[b].cpu().numpy(), scales=g.scales[b].cpu().numpy(),
                                  idx_codes=g.idx_codes[b].cpu().numpy(),
                                  idx_scale=g.idx_scale[b].cpu().numpy()))
        for r in st.swa:
            out["swa"].append(dict(codes=r.codes[b].cpu().numpy(), scale=r.scale[b].cpu().numpy()))
        for l, t in st.topk.items():
            out["topk"][l] = t[b].cpu().numpy()
            out["count"][l] = st.count[l][b].cpu().numpy()
        for g, p in st.pool.items():
            out["pool"][g] = p[b].cpu().numpy()
        for l in range(len(st.plan)):
            out["out"].append(st.out[l][b].cpu().numpy())
            out["lse"].append(st.lse[l][b].cpu().numpy())
        return out
