"""Host-side logic of bench.py: the multi-rank path on two gloo ranks (CPU), the
algorithmic byte counts, and the reference arm's output line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from synth.workloads import WORKLOADS  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        wl = bench.rank_workload(WORKLOADS["decode_128k"], rank)
        first = wl.q_idx_batch(0)[0, 0, 0, :8].view(torch.int16).tolist()
        out.put((rank, ms, wl.b0, wl.B, wl.name, first,
                 bench.job_value(world, len(wl.layers), ms)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_disjoint_requests():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, b00, B0, n0, f0, v0), (r1, ms1, b01, B1, n1, f1, v1) = res
    assert ms0 == ms1 == 15.0                  # both ranks time the slowest rank
    assert (b00, b01) == (0, 64) and B0 == B1 == 64 and n0 == n1 == "decode_128k"
    # rank 1's first request is global request 64, not a copy of rank 0's
    ref = WORKLOADS["decode_128k"]
    assert f1 == ref.q_idx(0, 64)[0, 0, :8].view(torch.int16).tolist()
    assert f0 != f1
    assert v0 == v1 == 2 * 20 / 0.015          # whole-job layer-steps/s


def test_algorithmic_bytes_at_128k():
    """Per-unit costs: 132 B of indexer K + 4 B score written + 4 B read back + block
    max per visible position; 288 B per selected entry and 516 B per window row."""
    wl = WORKLOADS["decode_128k"]
    ob = bench.op_bytes(wl)
    N, B = 131072, 64
    nb = N // 8
    per_q = (N * 132 + 4 * N + 4 * nb + 4 * nb + 8 * 2048 * 4 + 4 * 2048 + 4 * 512 + 4
             + 4 * 128 * 2 + 4 * 4)
    assert ob["index_full_g0"] == B * per_q == 1_154_155_776
    attn = 512 * 288 + 512 * 4 + 128 * 516 + 64 * 512 * 2 + 64 * 512 * 4 + 64 * 4
    assert ob["attn"] == B * attn
    # Reindex: the pool, 8 entries of index K (128 B codes + 4 B scale) per pool block, the
    # scores and slot maxima written, the maxima read, the top_k chosen slots' scores read
    # back, the Top-K out
    rx = (4 * 2048 + 8 * 2048 * 132 + 8 * 2048 * 4 + 4 * 2048 * 2 + 8 * 512 * 4 + 4 * 512 + 4
          + 4 * 128 * 2 + 4 * 4)
    assert ob["index_reindex_g0"] == B * rx == 145_425_664
    assert bench.step_bytes(wl) == 2_265_830_912


def test_reference_arm_line():
    """`--impl reference` times the CPU oracle and prints one line with impl=reference."""
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_full_layer", "--steps", "1", "--warmup", "1"],
                       capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["unit"] == bench.UNIT


def test_reference_arm_other_ranks_do_nothing():
    class A:
        workload = "decode_128k"
        steps = 1
    assert bench.run_reference(A(), 1, 2) is None


def test_op_rooflines_dominant_and_traffic():
    """Per-op roofline entries: algorithmic bytes per step over the op's measured time per
    step (the per-call intervals partition the step, so the shares add up to 1), ncu
    traffic only while the captured kernel's sources are unchanged, dominant op by share."""
    from fp4_kv_compressed_b200.stack import plan_layers
    wl = WORKLOADS["decode_128k"]
    plan = plan_layers([g.schedule for g in wl.groups])
    # the ordinary calls: 19 fused attention launches, 4 Reindex ops
    per = bench.op_step_bytes(wl, plan, reuse=False)
    assert per["csa2_quantize_append"][1] == 1 and per["csa2_index_full"][1] == 1
    assert per["csa2_index_reindex"][1] == 4 and per["csa2_sparse_attn_decode"][1] == 1
    assert per["csa2_sparse_attn_decode_append"][1] == 19
    assert sum(b for b, _ in per.values()) == bench.step_bytes(wl)
    # the stack's default: the 15 Reuse layers and the 4 Reindex ops overlap their
    # predecessors through their own calls; the same bytes in all
    per_r = bench.op_step_bytes(wl, plan)
    assert per_r["csa2_sparse_attn_decode_reuse"][1] == 15 and per_r["csa2_sparse_attn_decode_append"][1] == 4
    assert per_r["csa2_index_reindex_settled"][1] == 4 and "csa2_index_reindex" not in per_r
    assert per_r["csa2_sparse_attn_decode_reuse"][0] == 15 * per["csa2_sparse_attn_decode_append"][0] // 19
    assert sum(b for b, _ in per_r.values()) == bench.step_bytes(wl)
    # paged caches: every call in its _paged form, the same bytes and launches
    per_p = bench.op_step_bytes(wl, plan, paged=True)
    assert set(per_p) == {"csa2_quantize_append_paged", "csa2_index_full_paged", "csa2_index_reindex_paged_settled",
                          "csa2_sparse_attn_decode_paged", "csa2_sparse_attn_decode_paged_reuse"}
    assert per_p["csa2_sparse_attn_decode_paged_reuse"][1] == 15 and per_p["csa2_sparse_attn_decode_paged"][1] == 5
    assert per_p["csa2_index_reindex_paged_settled"][1] == 4
    assert bench.op_step_bytes(wl, plan, reuse=False, paged=True)["csa2_index_reindex_paged"][1] == 4
    assert sum(b for b, _ in per_p.values()) == bench.step_bytes(wl)
    assert sum(n for _, n in per_p.values()) == sum(n for _, n in per.values())
    op_ms = {"csa2_quantize_append": (0.005, 1), "csa2_index_full": (0.4, 1),
             "csa2_index_reindex": (0.4, 4), "csa2_sparse_attn_decode": (0.03, 1),
             "csa2_sparse_attn_decode_append": (0.665, 19)}
    ms_step = sum(t for t, _ in op_ms.values())
    ops = bench.op_rooflines(wl, plan, op_ms, ms_step=ms_step, reuse=False)
    assert abs(sum(e["share_of_step"] for e in ops.values()) - 1.0) < 1e-12
    f = ops["csa2_index_full"]
    assert f["launches_per_step"] == 1 and f["bound"] == "hbm"
    assert abs(f["achieved"] - 1_154_155_776 / 0.4e-3 / 1e9) < 1e-6
    a = ops["csa2_sparse_attn_decode_append"]
    assert a["launches_per_step"] == 19 and abs(a["launch_ms"] - 0.035) < 1e-12
    assert a["algorithmic_bytes_per_launch"] == bench.op_bytes(wl)["attn"] + 64 * (1024 + 516)
    assert a["tensor"]["flops_per_launch"] == 64 * 4 * 64 * 512 * 640
    assert ops["csa2_index_reindex"]["launches_per_step"] == 4
    for name, e in ops.items():
        caps, files, sha = bench.NCU_TRAFFIC.get(name, ([], (), ""))
        expect = (sum(tb * wl.B / b for tb, b in caps)
                  if caps and bench._sources_hash(files) == sha else None)
        assert e["traffic"] == expect
    assert max(ops, key=lambda n: ops[n]["share_of_step"]) == "csa2_sparse_attn_decode_append"


def test_code_hash_ignores_comments_only():
    """The traffic key follows the code, not its comments."""
    import bench
    a = b"int f(int x) {  // doubles\n    return 2 * x;\n}\n"
    b = b"// a new header line\nint f(int x) {  // twice x\n\n    return 2 * x;\n}\n"
    c = b"int f(int x) {\n    return 3 * x;\n}\n"
    assert bench.code_hash(a) == bench.code_hash(b) != bench.code_hash(c)


def test_prefill_and_rope_op_rooflines():
    """The prefill chunk's tensor-core Full op: the index cache is read once per request
    (not once per query token), its tensor flops are 2 * H_I * d per (query, visible
    entry), and no decode traffic capture is scaled onto it.  The RoPE attention op adds
    one (cos, sin) table row per query."""
    from fp4_kv_compressed_b200.stack import plan_layers
    from synth.workloads import ROPE_PAIRS
    wl = WORKLOADS["prefill_chunk_enc"]
    N, d, HI, Tq = wl.entries(0), wl.d_I, wl.H_I, wl.Tq
    ob = bench.op_bytes(wl)
    assert ob["index_full_g0"] == N * (d + 4) + Tq * (8 * N + 4 * wl.top_k + 4 + HI * d * 2 + HI * 4)
    vis = sum((t + 1) // 2 for t in range(wl.ctx - Tq, wl.ctx))
    assert bench.index_scan_flops(wl, 0) == vis * 2 * HI * d
    plan = plan_layers([g.schedule for g in wl.groups])
    ops = bench.op_rooflines(wl, plan, {"csa2_index_full_tc": (0.6, 1),
                                        "csa2_sparse_attn_decode": (4.2, 6)},
                             ms_step=4.7, index_scan="tc")
    tc = ops["csa2_index_full_tc"]
    assert tc["traffic"] is None and ops["csa2_sparse_attn_decode"]["traffic"] is None
    assert abs(tc["tensor"]["achieved"] - vis * 2 * HI * d / 0.6e-3 / 1e12) < 1e-9
    assert tc["bound"] == "hbm"          # the score round trip outweighs the MMAs
    dec = WORKLOADS["decode_128k"]
    plan = plan_layers([g.schedule for g in dec.groups])
    r = bench.op_rooflines(dec, plan, {"csa2_sparse_attn_decode_append_rope": (19 * 0.033, 19)}, 1.12,
                           rope=True, reuse=False)
    e = r["csa2_sparse_attn_decode_append_rope"]
    assert e["algorithmic_bytes_per_launch"] == (bench.op_bytes(dec)["attn"] + 64 * (1024 + 516)
                                                 + 64 * ROPE_PAIRS * 8)
    assert e["launches_per_step"] == 19 and e["traffic"] is None
