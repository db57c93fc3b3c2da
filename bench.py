"""Benchmark of the CSA2 decode path (one JSON line on rank 0).

A step = one decode token through the whole layer stack of the workload (every
row of the hot path: quantise-append, Full scan + pool + Top-K, Reindex, Reuse,
sparse attention) for the whole batch.  Metric: CSA2 decode layer-steps/s (a
layer-step = one layer for the whole batch).  Default workload: batch 64 at
context 131072, decoder stack F+4X+15U (decode_128k).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the CPU oracle as the reference arm)
  python bench.py --workload prefill_chunk_enc --index-scan tc
      (a 2048-token prefill chunk; the Full scan on the tensor cores)
  python bench.py --rope   (pre-RoPE rows, rotated inside the append launches)

Multi-GPU (torchrun): requests are independent, so each rank runs its own batch
with no collective on the data path (weak scaling); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "CSA2 decode layer-steps/s; indexer+attn HBM GB/s as % of 8 TB/s"
UNIT = "layer-steps/s"
HBM_FALLBACK_GBS = 6650.0


# ------------------------------------------------------------------------------------------
# algorithmic bytes (per op and per step)
# ------------------------------------------------------------------------------------------
def op_bytes(wl) -> dict:
    """Bytes the method must move, per launch of each op (whole batch)."""
    B, Tq, d, HI, K = wl.B, wl.Tq, wl.d_I, wl.H_I, wl.top_k
    BT = B * Tq
    out = {}
    for g, grp in enumerate(wl.groups):
        N = wl.entries(g)
        nb = (N + 7) // 8
        q = HI * d * 2 + HI * 4
        if grp.pool_blocks:
            P = grp.pool_blocks
            per = (N * (d + 4) + 4 * N + 4 * nb + 4 * nb + 8 * min(P, nb) * 4 + 4 * P + 4 * K + 4
                   + q)
            out[f"index_full_g{g}"] = BT * per
            # the pool, its entries' index K and scales, the scores and slot maxima
            # written, the chosen slots' scores read back, the Top-K out
            rp = 4 * P + 8 * P * (d + 4) + 8 * P * 4 + 4 * P + 4 * P + 8 * K * 4 + 4 * K + 4 + q
            out[f"index_reindex_g{g}"] = BT * rp
        else:
            out[f"index_full_g{g}"] = BT * (N * (d + 4) + 4 * N + 4 * N + 4 * K + 4 + q)
        if Tq > 1:
            # the query tokens of a request share its index cache: read it once
            out[f"index_full_g{g}"] -= (BT - B) * N * (d + 4)
        out[f"append_g{g}"] = B * max(1, wl.entries(g) - wl.first_q_pos // grp.ratio) * (
            512 * 2 + 288 + d * 2 + d + 4)
    n_win = min(wl.swa_len, wl.first_q_pos + 1)
    out["attn"] = BT * (K * 288 + K * 4 + n_win * 516 + wl.H * 512 * 2 + wl.H * 512 * 4 + wl.H * 4)
    out["swa_append"] = B * Tq * (512 * 2 + 516)
    # RoPE inside the append: one (cos, sin) fp32 row of the table per rotated row
    from synth.workloads import ROPE_PAIRS
    out["rope_row"] = B * Tq * ROPE_PAIRS * 8
    return out


def index_scan_flops(wl, g: int) -> int:
    """Score products of a Full scan: 2 * H_I * d_idx flop per (query, visible entry)."""
    vis = sum(min((t + 1) // wl.groups[g].ratio, wl.entries(g)) for t in wl.q_positions())
    return wl.B * vis * 2 * wl.H_I * wl.d_I


def attn_flops(wl) -> int:
    """Q K^T and P V over the selection and the window: 4 * H * 512 flop per key."""
    n_win = min(wl.swa_len, wl.first_q_pos + 1)
    return wl.B * wl.Tq * 4 * wl.H * 512 * (wl.top_k + n_win)


# DRAM bytes (read + write) per launch from one ncu capture of each of an op's kernels
# in decode (one query token per request): ([(bytes, batch of the captured launch), ...],
# kernel sources, code_hash of those sources at capture time).  Reported, each kernel
# scaled to the batch, only for decode workloads and while the code is unchanged.
NCU_TRAFFIC = {
    # attention: attn_kernel<0, 2> (2 CTAs per query) at batch 40, one launch
    "csa2_sparse_attn_decode": ([(13_242_112, 40)], ("csa2_attn.cu",), "cf0d443258f3fd02"),
    "csa2_sparse_attn_decode_append": ([(13_242_112, 40)], ("csa2_attn.cu",), "cf0d443258f3fd02"),
    "csa2_sparse_attn_decode_reuse": ([(13_242_112, 40)], ("csa2_attn.cu",), "cf0d443258f3fd02"),
    # Full: index_scan_kernel + select_full_kernel at batch 8
    "csa2_index_full": ([(138_471_936 + 4_568_064, 8), (1_127_680, 8)], ("csa2_index.cu",),
                        "c796ebf0ae6d4c2b"),
    # Reindex: reindex_score_kernel + select_reindex_kernel at batch 8
    "csa2_index_reindex": ([(18_616_832, 8), (542_208, 8)], ("csa2_index.cu",), "c796ebf0ae6d4c2b"),
    "csa2_index_reindex_settled": ([(18_616_832, 8), (542_208, 8)], ("csa2_index.cu",), "c796ebf0ae6d4c2b"),
}


def code_hash(text: bytes) -> str:
    """sha256[:16] of a source with its // comments and blank lines removed, so that
    the key changes with the code but not with its comments."""
    import hashlib
    h = hashlib.sha256()
    for ln in text.decode().splitlines():
        code = ln.split("//", 1)[0].rstrip()
        if code:
            h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def _sources_hash(files) -> str:
    return code_hash(b"".join(open(os.path.join(ROOT, "fp4_kv_compressed_b200", "csrc", f), "rb").read()
                              for f in files))


def measured_peaks() -> dict:
    out = {"hbm_gbs": HBM_FALLBACK_GBS, "tflops": 1400.0, "source": "fallback (6.65 TB/s, 1.4 PF/s)"}
    try:
        mp = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        out = {"hbm_gbs": float(mp["hbm_gbs"]), "tflops": float(mp["bf16_tflops_sustained"]),
               "source": "of measured (MEASURED_PEAKS.json: hbm_gbs; bf16_tflops_sustained, "
                         "the kernels being timed inside a long step)"}
    except Exception:
        pass
    return out


OP_KERNELS = {
    "csa2_quantize_append": "quantize_append_kernel",
    "csa2_quantize_append_rope": "quantize_append_kernel",
    "csa2_index_full": "index_scan_kernel + select_full_kernel",
    "csa2_index_full_tc": "index_scan_tc_kernel + select_full_kernel",
    "csa2_index_reindex": "reindex_score_kernel + select_reindex_kernel",
    "csa2_index_reindex_settled": "reindex_score_kernel (overlapping the previous launch) + select_reindex_kernel",
    "csa2_sparse_attn_decode": "attn_kernel",
    "csa2_sparse_attn_decode_reuse": "attn_kernel (Reuse layer, with the SWA append, overlapping the previous launch)",
    "csa2_sparse_attn_decode_append": "attn_kernel (with the SWA append)",
    "csa2_sparse_attn_decode_append_rope": "attn_kernel (with the RoPE + SWA append)",
    "csa2_quantize_append_paged": "quantize_append_kernel (paged cache)",
    "csa2_index_full_paged": "index_scan_kernel + select_full_kernel (paged cache)",
    "csa2_index_reindex_paged": "reindex_score_kernel + select_reindex_kernel (paged cache)",
    "csa2_sparse_attn_decode_paged": "attn_kernel (paged cache; with the SWA append in decode)",
    "csa2_index_reindex_paged_settled": "reindex_score_kernel (paged cache, overlapping the previous launch) + "
                                        "select_reindex_kernel",
    "csa2_sparse_attn_decode_paged_reuse": "attn_kernel (paged cache, Reuse layer, with the SWA append, "
                                           "overlapping the previous launch)",
}


def op_step_bytes(wl, plan, rope: bool = False, index_scan: str = "exact", reuse: bool = True,
                  paged: bool = False) -> dict:
    """Per library call name: (algorithmic bytes per step, launches per step), walking the
    layer plan the way DecodeStack.step issues its calls (reuse: DecodeStack.reuse_launch,
    the Reuse and Reindex layers' overlapping calls; paged: the caches in pages, every
    call in its _paged form, the same bytes)."""
    if paged:
        out = {}
        for name, v in op_step_bytes(wl, plan, rope, index_scan, reuse).items():
            if name == "csa2_sparse_attn_decode_reuse":
                name = "csa2_sparse_attn_decode_paged_reuse"
            elif name.startswith("csa2_sparse_attn_decode"):
                name = "csa2_sparse_attn_decode_paged"
            elif name.startswith("csa2_quantize_append"):
                name = "csa2_quantize_append_paged"
            elif name == "csa2_index_reindex_settled":
                name = "csa2_index_reindex_paged_settled"
            else:
                name += "_paged"
            b, n = out.get(name, (0, 0))
            out[name] = (b + v[0], n + v[1])
        return out
    ob = op_bytes(wl)
    fused = wl.Tq == 1 and wl.swa_len > 0          # decode: SWA append inside the attention
    first = {}
    for lp in plan:
        first.setdefault(lp.group, lp.layer)
    app = "csa2_quantize_append_rope" if rope else "csa2_quantize_append"
    full = "csa2_index_full_tc" if index_scan == "tc" else "csa2_index_full"
    out = {}

    def add(name, nbytes):
        b, n = out.get(name, (0, 0))
        out[name] = (b + nbytes, n + 1)
    for lp in plan:
        g = lp.group
        if lp.layer == first[g]:
            add(app, ob[f"append_g{g}"] + ob["swa_append"])
        elif not fused:
            add(app, ob["swa_append"])
        if lp.mode == "F":
            add(full, ob[f"index_full_g{g}"])
        elif lp.mode == "X":
            add("csa2_index_reindex_settled" if reuse else "csa2_index_reindex", ob[f"index_reindex_g{g}"])
        if fused and lp.layer != first[g]:
            if reuse and lp.mode == "U":
                name = "csa2_sparse_attn_decode_reuse"
            else:
                name = "csa2_sparse_attn_decode_append" + ("_rope" if rope else "")
            add(name, ob["attn"] + ob["swa_append"] + (ob["rope_row"] if rope else 0))
        else:
            add("csa2_sparse_attn_decode", ob["attn"])
    return out


def op_rooflines(wl, plan, op_ms: dict, ms_step: float, rope: bool = False,
                 index_scan: str = "exact", reuse: bool = True, paged: bool = False) -> dict:
    """Per library call: algorithmic bytes (and flops) per step over its measured time per
    step.  op_ms[name] = (total ms per step of the calls of that name, calls per step)."""
    pk = measured_peaks()
    per = op_step_bytes(wl, plan, rope, index_scan, reuse, paged)
    modes = [lp.mode for lp in plan]
    out = {}
    for name, (tot_ms, n) in op_ms.items():
        nbytes_step, n_plan = per.get(name, (0, 0))
        if not nbytes_step or not n:
            continue
        ms = tot_ms / n
        gbs = nbytes_step / (tot_ms / 1e3) / 1e9
        traffic = None
        if name in NCU_TRAFFIC:
            caps, files, sha = NCU_TRAFFIC[name]
            if caps and _sources_hash(files) == sha and wl.Tq == 1:
                traffic = sum(tb * wl.B / tbatch for tb, tbatch in caps)
        e = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
             "frac": gbs / pk["hbm_gbs"], "traffic": traffic, "kernels": OP_KERNELS.get(name, name),
             "algorithmic_bytes_per_launch": nbytes_step / n_plan, "launch_ms": ms,
             "launches_per_step": n, "share_of_step": tot_ms / ms_step, "peak_source": pk["source"]}
        fl = None
        if name.startswith("csa2_sparse_attn_decode"):
            fl = attn_flops(wl) * n
        elif name == "csa2_index_full_tc":
            fl = sum(index_scan_flops(wl, lp.group) for lp in plan if lp.mode == "F")
        if fl:
            tfs = fl / (tot_ms / 1e3) / 1e12
            e["tensor"] = {"achieved": tfs, "peak": pk["tflops"], "unit": "TFLOP/s",
                           "frac": tfs / pk["tflops"], "flops_per_launch": fl / n}
            if fl / (pk["tflops"] * 1e12) > nbytes_step / (pk["hbm_gbs"] * 1e9):
                e.update(bound="tensor", achieved=tfs, peak=pk["tflops"], unit="TFLOP/s",
                         frac=tfs / pk["tflops"])
        out[name] = e
    return out


def step_bytes(wl) -> int:
    ob = op_bytes(wl)
    total = 0
    for g, grp in enumerate(wl.groups):
        total += ob[f"append_g{g}"]
        for m in grp.schedule:
            total += ob["attn"] + ob["swa_append"]
            if m == "F":
                total += ob[f"index_full_g{g}"]
            elif m == "X":
                total += ob[f"index_reindex_g{g}"]
    return total


# ------------------------------------------------------------------------------------------
# ranks: disjoint requests per rank, time = max over ranks
# ------------------------------------------------------------------------------------------
def rank_workload(wl, rank: int):
    """Rank r holds global requests r*B .. r*B + B - 1 (requests are independent: weak
    scaling with no collective on the data path)."""
    from synth.workloads import small_variant
    return small_variant(wl, b0=wl.b0 + rank * wl.B, name=wl.name) if rank else wl


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, layers: int, ms_step: float) -> float:
    """Whole-job layer-steps/s: every rank runs `layers` layer-steps per step."""
    return world * layers / (ms_step / 1e3)


# ------------------------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ------------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.ok = [], set(), False
        self._stop = threading.Event()
        try:
            import pynvml as N
            import torch
            N.nvmlInit()
            p = torch.cuda.get_device_properties(device_index)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            try:
                self.h = N.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = N.nvmlDeviceGetHandleByIndex(device_index)
            self.N = N
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report nothing rather than guess
            self.err = str(e)

    def _run(self):
        N = self.N
        while not self._stop.is_set():
            try:
                self.samples.append(N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM))
                r = N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self) -> dict:
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------
# CPU oracle sample (cpu_baseline leg and the reference arm)
# ------------------------------------------------------------------------------------------
def oracle_sample_time(wl, requests: list[int], steps: int = 1) -> tuple[float, dict]:
    """Time the oracle on one decode step of `requests` (caches prepared untimed).
    Returns seconds per step for those requests and a description."""
    import torch
    import oracle as orc
    from oracle import workload_ref as R

    prepared = []
    for b in requests:
        caches = R.request_caches(wl, b, main_rows={g: np.zeros(0, np.int64)
                                                    for g in range(len(wl.groups))})
        for g, c in enumerate(caches):   # main KV of the whole request (state before the step)
            N = c["N"]
            mc, ms = orc.quantize_fp4(wl.main_kv(g, b, 0, N))
            c["codes"], c["scales"] = mc, ms
        rings = [R.swa_ring(wl, l, b) for l in range(len(wl.layers))]
        inputs = dict(q=[wl.q(l, b) for l in range(len(wl.layers))],
                      qi=[wl.q_idx(l, b) for l in range(len(wl.layers))],
                      w=[wl.w(l, b).numpy() for l in range(len(wl.layers))],
                      kv=[wl.main_kv(g, b, wl.entries(g) - 1, 1) for g in range(len(wl.groups))],
                      ik=[wl.idx_k(g, b, wl.entries(g) - 1, 1) for g in range(len(wl.groups))],
                      swa=[wl.swa(l, b, wl.ctx - 1, 1) for l in range(len(wl.layers))])
        prepared.append((b, caches, rings, inputs))
    q_pos = np.asarray(wl.q_positions(), np.int32)[None]
    plan = R.reuse_sources(wl)
    t0 = time.perf_counter()
    for _ in range(steps):
        for b, caches, rings, inp in prepared:
            for g in range(len(wl.groups)):           # a1/a2: the new entry
                orc.quantize_fp4(inp["kv"][g])
                orc.quantize_fp8(inp["ik"][g])
            topk, pool = {}, {}
            for layer, (g, m, src) in enumerate(plan):
                c, grp = caches[g], wl.groups[g]
                orc.quantize_fp8(inp["swa"][layer])    # a2: this layer's SWA row
                if m == "F":
                    p, t, _ = orc.index_full(c["idx_codes"][None], c["idx_scale"][None], grp.ratio,
                                             inp["qi"][layer][None], inp["w"][layer][None], q_pos,
                                             grp.pool_blocks, wl.top_k)
                    topk[layer], pool[g] = t, p
                elif m == "X":
                    t, _ = orc.index_reindex(c["idx_codes"][None], c["idx_scale"][None],
                                             grp.ratio, inp["qi"][layer][None],
                                             inp["w"][layer][None], q_pos, pool[g], wl.top_k)
                    topk[layer] = t
                rc, rs = rings[layer]
                orc.attention(c["codes"][None], c["scales"][None], rc[None], rs[None],
                              inp["q"][layer][None], q_pos, topk[src], wl.swa_len, R.SOFTMAX_SCALE)
    dt = (time.perf_counter() - t0) / steps
    return dt, {"requests": len(requests), "of_batch": wl.B, "steps": steps}


def cpu_baseline(wl, requests: list[int]) -> dict:
    import oracle as orc
    dt, desc = oracle_sample_time(wl, requests, 1)
    layers = len(wl.layers)
    value = layers * len(requests) / wl.B / dt
    return {"value": value, "unit": UNIT, "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"{len(requests)} of {wl.B} requests, 1 decode step of all {layers} layers "
                      f"(append, index, attention) on the host; value scaled by "
                      f"{len(requests)}/{wl.B} of a layer-step; {dt:.2f} s per sample step"}


# ------------------------------------------------------------------------------------------
def pack_inputs(inputs: dict, device):
    """Copy every step input into one device buffer (views replace the tensors) and
    return (views dict, device buffer, pinned host mirror, bytes)."""
    import torch
    flat = []

    def visit(v):
        if torch.is_tensor(v):
            flat.append(v)
        elif isinstance(v, (list, tuple)):
            for x in v:
                visit(x)
    for v in inputs.values():
        visit(v)
    offs, off = [], 0
    for t in flat:
        off = (off + 255) // 256 * 256
        offs.append(off)
        off += t.numel() * t.element_size()
    dbuf = torch.empty(off, dtype=torch.uint8, device=device)
    views = {}
    for t, o in zip(flat, offs):
        n = t.numel() * t.element_size()
        v = dbuf[o:o + n].view(t.dtype).view(t.shape)
        v.copy_(t)
        views[id(t)] = v

    def rebuild(v):
        if torch.is_tensor(v):
            return views[id(v)]
        if isinstance(v, list):
            return [rebuild(x) for x in v]
        return v
    packed = {k: rebuild(v) for k, v in inputs.items()}
    hbuf = torch.empty(off, dtype=torch.uint8, pin_memory=True)
    hbuf.copy_(dbuf)
    return packed, dbuf, hbuf, off


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from synth.workloads import WORKLOADS
    import csa2_harness

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.workload]
    if args.batch:
        from synth.workloads import small_variant
        wl = small_variant(wl, B=args.batch, name=f"{wl.name}_b{args.batch}")
    wl = rank_workload(wl, rank)
    dw = csa2_harness.DeviceWorkload(wl, device=dev, index_scan=args.index_scan, rope=args.rope,
                                     page_size=args.page_size)
    st = dw.stack
    inputs, dbuf, hbuf, in_bytes = pack_inputs(dw.inputs, dev)
    full_layers = [lp.layer for lp in st.plan if lp.mode == "F"]
    stream = torch.cuda.Stream(device=dev)

    # one eager step (sets kernel attributes, checks the path), then the graph
    with torch.cuda.stream(stream):
        st.step(**inputs)
    torch.cuda.synchronize(dev)
    if st.dev_err.item() != 0:
        raise RuntimeError(f"device error bits {st.dev_err.item()} in the warm-up step")
    if args.profile_steps:
        # for profilers: warm-up steps, then the requested eager steps inside one NVTX
        # range named "step" (e.g. ncu --nvtx --nvtx-include "step/"); no timing
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                st.step(**inputs)
            torch.cuda.synchronize(dev)
            torch.cuda.nvtx.range_push("step")
            for _ in range(args.profile_steps):
                st.step(**inputs)
            torch.cuda.synchronize(dev)
            torch.cuda.nvtx.range_pop()
        return None, wl

    S = max(1, min(10, args.steps))
    import fp4_kv_compressed_b200.stack as stack_mod

    # The headline graph holds S steps and no events.  A second graph holds one step
    # with a CUDA event recorded on the launching stream after every library call (and
    # one before the first): consecutive events partition the step, so each call's
    # time is the interval between its two events and the calls' times add up to the
    # step.  It is replayed after the timed region, with the same warm-up and
    # synchronisation, for the per-op figures (roofline, shares).
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(S):
            st.step(**inputs)
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=stream):
        st.step(**inputs)
    op_names = [n for n in ("csa2_quantize_append", "csa2_quantize_append_rope", "csa2_index_full",
                            "csa2_index_full_tc", "csa2_index_reindex", "csa2_index_reindex_settled",
                            "csa2_sparse_attn_decode", "csa2_sparse_attn_decode_append",
                            "csa2_sparse_attn_decode_append_rope", "csa2_sparse_attn_decode_reuse",
                            "csa2_quantize_append_paged", "csa2_index_full_paged", "csa2_index_reindex_paged",
                            "csa2_sparse_attn_decode_paged", "csa2_index_reindex_paged_settled",
                            "csa2_sparse_attn_decode_paged_reuse")
                if hasattr(stack_mod.bind, n)]
    originals = {name: getattr(stack_mod.bind, name) for name in op_names}
    marks = []                       # (op name, event after the call)

    def make_marked(name):
        orig = originals[name]

        def f(*a, **k):
            orig(*a, **k)
            e = torch.cuda.Event(enable_timing=True, external=True)
            e.record()
            marks.append((name, e))
        return f

    g_ops = torch.cuda.CUDAGraph()
    for name in op_names:
        setattr(stack_mod.bind, name, make_marked(name))
    try:
        with torch.cuda.graph(g_ops, stream=stream):
            e_first = torch.cuda.Event(enable_timing=True, external=True)
            e_first.record()
            st.step(**inputs)
    finally:
        for name, orig in originals.items():
            setattr(stack_mod.bind, name, orig)

    reps = max(1, args.steps // S)
    K = reps * S
    for _ in range(max(args.warmup, 3)):
        g1.replay()
    torch.cuda.synchronize(dev)

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with clocks:
        with torch.cuda.stream(stream):
            start.record()
            for _ in range(reps):
                g.replay()
            end.record()
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms = start.elapsed_time(end)
    # per-op figures from the partitioned graph (replayed after the timed region)
    op_sum, op_n, ops_step = {}, {}, []
    for _ in range(max(args.warmup, 3)):
        g_ops.replay()
    torch.cuda.synchronize(dev)
    for _ in range(max(3, min(20, reps))):
        with torch.cuda.stream(stream):
            g_ops.replay()
        torch.cuda.synchronize(dev)
        prev, tot = e_first, 0.0
        for name, e in marks:
            dt = prev.elapsed_time(e)
            op_sum[name] = op_sum.get(name, 0.0) + dt
            op_n[name] = op_n.get(name, 0) + 1
            prev, tot = e, tot + dt
        ops_step.append(tot)
    n_rep = len(ops_step)
    op_ms = {name: (op_sum[name] / n_rep, op_n[name] // n_rep) for name in op_sum}
    ops_step_ms = statistics.mean(ops_step)
    ms_max = max_over_ranks(ms, world, dev)
    if st.dev_err.item() != 0:
        raise RuntimeError(f"device error bits {st.dev_err.item()} in the timed steps")

    # ---- e2e: inputs from pinned host memory, last layer's output back to the host ----
    # Every step copies its inputs host -> device and its result device -> host.  The
    # inputs are double-buffered: while step k computes on one device buffer, a copy
    # stream fills the other with step k + 1's inputs (the way a serving loop overlaps
    # its transfers), so the step costs max(copy, compute) rather than their sum.
    last = len(st.plan) - 1
    out_h = torch.empty_like(st.out[last], device="cpu").pin_memory()
    lse_h = torch.empty_like(st.lse[last], device="cpu").pin_memory()
    out_bytes = out_h.numel() * 4 + lse_h.numel() * 4
    Ke = 0 if args.no_e2e else max(3, min(K, args.e2e_steps))
    e2e_ms = None
    if Ke:
        inputs_b, dbuf_b, _, _ = pack_inputs(dw.inputs, dev)
        g1b = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1b, stream=stream):
            st.step(**inputs_b)
        bufs, graphs = (dbuf, dbuf_b), (g1, g1b)
        copy_stream = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event(), torch.cuda.Event()]
        free = [torch.cuda.Event(), torch.cuda.Event()]
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)

        def run(n, timed):
            for e in free:                                # both buffers free at the start
                e.record(stream)
            if timed:
                e0.record(copy_stream)
            for k in range(n):
                j = k % 2
                with torch.cuda.stream(copy_stream):      # step k's inputs, host -> device
                    copy_stream.wait_event(free[j])
                    bufs[j].copy_(hbuf, non_blocking=True)
                    copied[j].record(copy_stream)
                with torch.cuda.stream(stream):
                    stream.wait_event(copied[j])
                    graphs[j].replay()
                    out_h.copy_(st.out[last], non_blocking=True)   # the step's result, device -> host
                    lse_h.copy_(st.lse[last], non_blocking=True)
                    free[j].record(stream)
            if timed:
                e1.record(stream)
        run(2, False)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        run(Ke, True)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / Ke

    layers = len(st.plan)
    ms_step = ms_max / K
    value = job_value(world, layers, ms_step)
    sb = step_bytes(wl)
    ob = op_bytes(wl)
    g_full = st.plan[full_layers[0]].group
    ops = op_rooflines(wl, st.plan, op_ms, ops_step_ms, rope=args.rope, index_scan=args.index_scan,
                       reuse=st.reuse_launch, paged=st.page_size > 0)
    dominant = max(ops, key=lambda n: ops[n]["share_of_step"])
    launches = st.launches_per_step() * K
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": ("bf16 MMA index (fp32 accumulate)" if args.index_scan == "tc" else "fp32 index")
                 + " / bf16+fp16 MMA attention",
        "data": "synthetic",
        "config": workload_config(wl, args, world),
        "step": {"cuda_graph": True, "algorithmic_bytes": sb,
                 "ms_with_op_events": ops_step_ms,
                 "gbps": sb / (ms_step / 1e3) / 1e9, "frac_of_8tbs": sb / (ms_step / 1e3) / 8e12,
                 "token_layer_steps_per_s": value * wl.B},
        "roofline": dict(ops[dominant], op=dominant),
        "roofline_ops": ops,
        "e2e": ({"value": job_value(world, layers, e2e_ms), "unit": UNIT,
                 "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes,
                 "ms_per_step": e2e_ms} if Ke else None),
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    return line, wl


def run_cp(args) -> dict:
    """Context parallel (one long request's entries split over shards), its S shards
    emulated in turn on one GPU: one decode step's Full layer and attention of the
    workload's hierarchical (decoder) group.  Device times (CUDA events around a CUDA
    graph of each call, median of --steps replays after --warmup) of each shard's slice
    scan with its local selections, of the merge, of each shard's partial attention and
    of the combine, beside the unsplit csa2_index_full and csa2_sparse_attn_decode on the
    same cache.  The two all-gathers between the steps need several GPUs and are not
    run; their bytes per step are reported."""
    import torch
    from synth.workloads import WORKLOADS
    import csa2_harness
    import fp4_kv_compressed_b200 as pkg
    from fp4_kv_compressed_b200 import _binding as bind
    from fp4_kv_compressed_b200.context_parallel import LibraryBackend as LB, slice_bounds

    S = args.cp_shards
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = WORKLOADS[args.workload]
    if args.batch:
        from synth.workloads import small_variant
        wl = small_variant(wl, B=args.batch, name=f"{wl.name}_b{args.batch}")
    dw = csa2_harness.DeviceWorkload(wl, device=dev)
    st = dw.stack
    dw.step()                                   # this step's entries and rows appended
    torch.cuda.synchronize(dev)
    lp = next(lp for lp in st.plan if lp.mode == "F" and dw.groups[lp.group].pool_blocks > 0)
    g, L = lp.group, lp.layer
    kv = st.kv[g]
    inp = dw.inputs
    B, Tq, H, H_I, K, W = wl.B, wl.Tq, wl.H, wl.H_I, wl.top_k, wl.swa_len
    P = dw.groups[g].pool_blocks
    N = wl.entries(g)
    q_pos, q_idx, w, q = inp["q_pos"], inp["q_idx"][L], inp["w"][L], inp["q"][L]
    ring = st.swa[L]
    scale = 1 / math.sqrt(512)
    err = st.dev_err
    stream = torch.cuda.Stream(device=dev)
    i32 = dict(dtype=torch.int32, device=dev)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > L2: written before every replay

    def timed(fn) -> float:
        with torch.cuda.stream(stream):
            fn()                                # eager once (kernel attributes)
        torch.cuda.synchronize(dev)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            fn()
        for _ in range(max(args.warmup, 3)):
            gr.replay()
        torch.cuda.synchronize(dev)
        ev = []
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                flush.zero_()
                e0.record(stream)
                gr.replay()
                e1.record(stream)
                ev.append((e0, e1))
        torch.cuda.synchronize(dev)
        return statistics.median(a.elapsed_time(b) for a, b in ev)

    # the unsplit calls
    pool = torch.empty(B, Tq, P, **i32)
    topk = torch.empty(B, Tq, K, **i32)
    cnt = torch.empty(B, Tq, **i32)
    ws = torch.empty(pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_FULL, B, Tq, N, 0, K, P), dtype=torch.uint8,
                     device=dev)
    out = torch.empty(B, Tq, H, 512, dtype=torch.float32, device=dev)
    lse = torch.empty(B, Tq, H, dtype=torch.float32, device=dev)
    t_full = timed(lambda: bind.csa2_index_full(kv.struct, q_idx, w, q_pos, Tq, H_I, N, P, K, pool, topk, cnt,
                                                ws, err, stream))
    t_attn = timed(lambda: bind.csa2_sparse_attn_decode(kv.struct, ring.struct, q, q_pos, Tq, H, topk, K, W,
                                                        scale, out, lse, None, err, stream))
    # the shards: copies of the slices of the cache
    bounds = slice_bounds(N, S)
    pool_lists = torch.zeros(S, B, Tq, P, dtype=torch.int64, device=dev)
    topk_lists = torch.zeros(S, B, Tq, K, dtype=torch.int64, device=dev)
    o_parts = torch.empty(S, B, Tq, H, 512, dtype=torch.float32, device=dev)
    l_parts = torch.empty(S, B, Tq, H, dtype=torch.float32, device=dev)
    t_slice, t_part, merged_ok = [], [], True
    t_merge = t_combine = 0.0
    shards = []
    for r, (lo, hi) in enumerate(bounds):
        kv_s = pkg.GlobalKV(B, max(hi - lo, 1), wl.d_I, kv.ratio, dev)
        for src, dst in ((kv.codes, kv_s.codes), (kv.scales, kv_s.scales), (kv.idx_codes, kv_s.idx_codes),
                         (kv.idx_scale, kv_s.idx_scale)):
            dst[:, :hi - lo].copy_(src[:, lo:hi])
        n_max = max(0, min(hi, (int(q_pos.max()) + 1) // kv.ratio) - lo)
        ws_s = torch.empty(max(256, pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_FULL, B, Tq, max(n_max, 1), 0,
                                                            K, P)), dtype=torch.uint8, device=dev)
        shards.append((kv_s, lo, hi, n_max, ws_s))
        t_slice.append(timed(lambda kv_s=kv_s, lo=lo, n_max=n_max, ws_s=ws_s, r=r: LB.index_full_slice(
            kv_s, lo, q_idx, w, q_pos, Tq, H_I, n_max, P, K, pool_lists[r], topk_lists[r], ws_s, err, stream))
            if n_max > 0 else 0.0)
    # the merge (every shard runs the same; shard 0's local range) and each shard's part
    gpool = torch.empty(B, Tq, P, **i32)
    gpool_loc = torch.empty(B, Tq, P, **i32)
    gtopk = torch.empty(B, Tq, K, **i32)
    gcnt = torch.empty(B, Tq, **i32)
    locs = [torch.empty(B, Tq, K, **i32) for _ in range(S)]
    BT = B * Tq

    def merge_calls(r):
        lo, hi = bounds[r]
        LB.index_merge(pool_lists, BT, S, P, P, lo // 8, -(-hi // 8), gpool, None, gpool_loc, stream)
        LB.index_merge(topk_lists, BT, S, K, K, lo, hi, gtopk, gcnt, locs[r], stream)

    t_merge = timed(lambda: merge_calls(0))
    for r in range(1, S):
        with torch.cuda.stream(stream):
            merge_calls(r)
    torch.cuda.synchronize(dev)
    merged_ok = bool(torch.equal(gtopk, topk) and torch.equal(gcnt, cnt) and torch.equal(gpool, pool))
    for r, (kv_s, lo, hi, n_max, ws_s) in enumerate(shards):
        win = r == S - 1
        t_part.append(timed(lambda kv_s=kv_s, r=r, win=win: LB.attention(
            kv_s, ring if win else None, q, q_pos, Tq, H, locs[r], K, W if win else 0, scale, o_parts[r],
            l_parts[r], err, stream)))
    out_c = torch.empty_like(out)
    lse_c = torch.empty_like(lse)
    t_combine = timed(lambda: LB.combine(o_parts, l_parts, S, B * Tq * H, out_c, lse_c, stream))
    torch.cuda.synchronize(dev)
    if st.dev_err.item() != 0:
        raise RuntimeError(f"device error bits {st.dev_err.item()}")
    diff = float(((out_c - out).norm(dim=-1) / out.norm(dim=-1).clamp_min(1e-30)).max())
    proj = max(t_slice) + t_merge + max(t_part) + t_combine
    return {
        "metric": "context-parallel Full layer + attention of one decode step, shards emulated on one GPU",
        "unit": "ms", "workload": wl.name, "group": g, "layer": L, "shards": S,
        "config": {"batch": B, "entries": N, "pool": P, "top_k": K, "heads": H, "swa": W,
                   "slices": [list(b) for b in bounds]},
        "unsplit_ms": {"csa2_index_full": t_full, "csa2_sparse_attn_decode": t_attn, "sum": t_full + t_attn},
        "slice_scan_ms": t_slice, "merge_ms": t_merge, "attention_part_ms": t_part, "combine_ms": t_combine,
        "projected_ms_per_gpu": proj,
        "all_gather_bytes_per_step": {"candidate_keys": S * B * Tq * (P + K) * 8,
                                      "partials": S * B * Tq * H * (512 + 1) * 4},
        "all_gathers": "not run: one GPU",
        "merged_equals_unsplit": merged_ok, "combined_max_row_diff_vs_unsplit": diff,
        "l2": "flushed (256 MB written) before every replay",
    }


def workload_config(wl, args, world: int) -> dict:
    """The `config` of a bench line: the workload and how it is run (the same for
    both arms)."""
    from synth.workloads import ROPE_PAIRS, ROPE_START
    ob = op_bytes(wl)
    g_full = next(g for g, grp in enumerate(wl.groups) if "F" in grp.schedule)
    return {"workload": wl.name, "batch_per_gpu": wl.B, "context": wl.ctx, "heads": wl.H,
            "index_heads": wl.H_I, "d_idx": wl.d_I, "top_k": wl.top_k,
            "pool": [g.pool_blocks for g in wl.groups],
            "schedule": [g.schedule for g in wl.groups], "swa": wl.swa_len,
            "query_tokens": wl.Tq, "index_scan": args.index_scan,
            "rope": ({"start": ROPE_START, "pairs": ROPE_PAIRS,
                      "rows": "main KV and SWA, rotated inside the append launches"}
                     if args.rope else None),
            "paged": ({"page_size": args.page_size, "pages": "each group's pool, handed to the requests "
                       "in a seeded random order"} if getattr(args, "page_size", 0) else None),
            "parallelism": f"replicas x{world} (requests sharded, no collective)",
            "l2": "inputs larger than L2: the Full scan streams "
                  f"{ob[f'index_full_g{g_full}'] / 1e9:.2f} GB per step"}


def run_reference(args, rank, world):
    from synth.workloads import WORKLOADS
    import oracle as orc
    wl = WORKLOADS[args.workload]
    if rank != 0:
        return None
    K = max(1, args.steps if args.steps <= 5 else 2)
    req = [0]
    oracle_sample_time(wl, req, 1)            # warm-up (OpenMP pools, page-in)
    dt, desc = oracle_sample_time(wl, req, K)
    layers = len(wl.layers)
    value = layers * len(req) / wl.B / dt
    sample = (f"{len(req)} of {wl.B} requests per step, {K} timed steps of all {layers} layers "
              f"on the host; value scaled by {len(req)}/{wl.B} of a layer-step")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": 1, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp32 index / fp64 attention", "data": "synthetic",
            "config": workload_config(wl, args, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": orc.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_128k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--index-scan", default="exact", choices=["exact", "tc"],
                    help="Full-layer scan: fixed fp32 order, or tensor cores (prefill chunks)")
    ap.add_argument("--rope", action="store_true",
                    help="pass pre-RoPE rows and rotate them inside the append launches")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (small cases for profiling)")
    ap.add_argument("--profile-steps", type=int, default=0,
                    help="run this many eager steps inside an NVTX range 'step' and exit (for ncu)")
    ap.add_argument("--page-size", type=int, default=0,
                    help="the caches in pages of this many entries (a power of two >= 256), shuffled")
    ap.add_argument("--cp-shards", type=int, default=0,
                    help="time the context-parallel calls with this many shards emulated on one GPU")
    args = ap.parse_args()
    if args.cp_shards:
        print(json.dumps(run_cp(args)), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line, wl = run_ours(args, rank, world, local_rank)
        if line is None:
            return
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(wl, [0, wl.B - 1])
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
