"""The seeded input generator: slices regenerate bit-identically, draws look like
their distributions, and the workloads have the shapes the pages give."""
import numpy as np
import torch

import synth
from synth.workloads import WORKLOADS


def test_slices_regenerate_identically():
    full = synth.rows_normal_bf16(5, "x", 3, 0, 100, 64)
    part = synth.rows_normal_bf16(5, "x", 3, 40, 10, 64)
    assert torch.equal(full[40:50].view(torch.int16), part.view(torch.int16))
    assert not torch.equal(full, synth.rows_normal_bf16(6, "x", 3, 0, 100, 64))


def test_distributions():
    x = synth.rows_normal_bf16(1, "n", 0, 0, 2000, 512).double()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1) < 0.01
    u = synth.rows_uniform_f32(1, "u", 0, 0, 1000, 512)
    assert float(u.min()) > 0 and float(u.max()) < 1 and abs(u.mean().item() - 0.5) < 0.01


def test_hash_has_no_int64_overflow():
    idx = torch.tensor([0, 1, (1 << 40) - 1, (1 << 39) + 12345], dtype=torch.int64)
    h = synth.hash_u32(idx, synth.tensor_keys(1, "t"))
    assert bool((h >= 0).all()) and bool((h <= 0xFFFFFFFF).all())


def test_workload_shapes():
    w4 = WORKLOADS["decode_128k"]
    assert w4.B == 64 and w4.ctx == 131072 and w4.H == 64 and w4.top_k == 512
    assert w4.groups[0].pool_blocks * 8 == 16384 and w4.swa_len == 128
    assert [m for _, m in w4.layers].count("X") == 4 and len(w4.layers) == 20
    w5 = WORKLOADS["decode_1m"]
    assert len(w5.layers) == 38 and w5.entries(0) == 1 << 19 and w5.entries(3) == 1 << 20
    w3 = WORKLOADS["prefill_chunk_enc"]
    assert w3.first_q_pos == 65536 and w3.entries(0) == (65536 + 2048) // 2
    assert w3.window_cap >= 128 + 2048 - 1
    s = w4._scale("cpu")
    assert float(s.min()) >= 0.25 and float(s.max()) <= 4.0


def test_request_offset_selects_global_requests():
    """A workload copy with b0 = k holds global requests k.. : its batch rows, per-request
    rows and planted rows equal those of the first workload's requests k.."""
    from synth.workloads import WORKLOADS, small_variant
    base = small_variant(WORKLOADS["decoder_group_32k"], B=4, ctx=2000)
    part = small_variant(base, B=2, b0=2)
    assert torch.equal(part.main_kv_batch(0, 10, 3), base.main_kv_batch(0, 10, 3)[2:])
    assert torch.equal(part.idx_k_batch(0, 0, 2000), base.idx_k_batch(0, 0, 2000)[2:])
    assert torch.equal(part.q_batch(4), base.q_batch(4)[2:])
    assert torch.equal(part.q_idx_batch(0), base.q_idx_batch(0)[2:])
    assert torch.equal(part.w_batch(4), base.w_batch(4)[2:])
    assert torch.equal(part.swa_batch(7, 5, 4), base.swa_batch(7, 5, 4)[2:])
    assert torch.equal(part.idx_k(0, 1, 0, 2000), base.idx_k(0, 3, 0, 2000))
    assert part.planted_rows(1)[0] == base.planted_rows(3)[0]
    assert part.planted_rows(0)[0] != base.planted_rows(0)[0]
