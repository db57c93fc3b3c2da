"""Host-side checks of the C ABI (no GPU): the library loads, exports every symbol
include/csa2.h declares, sizes its workspaces, and rejects bad arguments before
any CUDA call.  Also the layer-schedule planner."""
import ctypes as C
import os
import re

import pytest

from conftest import ROOT


def header_functions() -> list[str]:
    src = open(os.path.join(ROOT, "include", "csa2.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(csa2_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def pkg():
    import fp4_kv_compressed_b200 as p
    return p


def test_library_exports_every_declared_symbol(pkg):
    lib = pkg.load_library()
    names = header_functions()
    assert set(names) == set(pkg.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n
    assert lib.csa2_abi_version() == 106      # 1.6: the paged forms of the overlapping launches
    for st in range(7):
        assert lib.csa2_status_string(st)


def test_workspace_sizes(pkg):
    ws = pkg.csa2_workspace_size
    full = ws(pkg.CSA2_OP_INDEX_FULL, 64, 1, 131072, 64, 512, 2048)
    assert full >= 64 * 131072 * 4 + 64 * 16384 * 4 and full % 256 == 0
    # long flat rows also hold the 8- and 64-position maxima; hierarchical rows hold the
    # 64-position maxima only beyond 16384 blocks
    flat = ws(pkg.CSA2_OP_INDEX_FULL, 64, 1, 131072, 64, 512, 0)
    assert flat >= 64 * 131072 * 4 + 64 * 16384 * 4 + 64 * 2048 * 4 and flat > full
    assert full == 64 * 131072 * 4 + 64 * 16384 * 4
    big = ws(pkg.CSA2_OP_INDEX_FULL, 4, 1, 1 << 20, 64, 512, 2048)
    assert big == 4 * (1 << 20) * 4 + 4 * (1 << 17) * 4 + 4 * (1 << 14) * 4
    short = ws(pkg.CSA2_OP_INDEX_FULL, 64, 1, 16384, 64, 512, 0)
    assert 64 * 16384 * 4 <= short < ws(pkg.CSA2_OP_INDEX_FULL, 64, 1, 16384, 64, 512, 2048)
    assert ws(pkg.CSA2_OP_INDEX_REINDEX, 64, 1, 0, 64, 512, 2048) >= 64 * 2048 * (8 + 1) * 4
    assert ws(pkg.CSA2_OP_SPARSE_ATTN, 64, 1, 0, 64, 512, 0) == 0
    assert ws(99, 1, 1, 1, 1, 1, 1) == 0


def test_validation_rejects_before_launch(pkg):
    lib = pkg.load_library()
    # null global-KV descriptor
    assert lib.csa2_index_full(None, None, None, None, 1, 4, 10, 0, 8, None, None, None, None,
                               0, None, None) == 1
    kv = pkg.CSA2GlobalKV(256, 256, 256, 256, 1, 100, 128, 1)
    qbuf = C.c_void_p(4096)
    # unsupported H_I, top_k and pool sizes
    assert lib.csa2_index_full(C.byref(kv), qbuf, qbuf, qbuf, 1, 3, 10, 0, 8, None, qbuf, qbuf,
                               qbuf, 1 << 20, None, None) == 4
    assert lib.csa2_index_full(C.byref(kv), qbuf, qbuf, qbuf, 1, 4, 10, 0, 513, None, qbuf, qbuf,
                               qbuf, 1 << 20, None, None) == 4
    assert lib.csa2_index_full(C.byref(kv), qbuf, qbuf, qbuf, 1, 4, 10, 256, 512, None, qbuf,
                               qbuf, qbuf, 1 << 20, None, None) == 4
    # workspace too small
    assert lib.csa2_index_full(C.byref(kv), qbuf, qbuf, qbuf, 1, 4, 100, 0, 8, None, qbuf, qbuf,
                               qbuf, 16, None, None) == 3
    # tensor-core Full scan: same checks, and q_idx must be 16-byte aligned
    assert lib.csa2_index_full_tc(C.byref(kv), qbuf, qbuf, qbuf, 1, 3, 10, 0, 8, None, qbuf,
                                  qbuf, qbuf, 1 << 20, None, None) == 4
    assert lib.csa2_index_full_tc(C.byref(kv), qbuf, qbuf, qbuf, 1, 4, 100, 0, 8, None, qbuf,
                                  qbuf, qbuf, 16, None, None) == 3
    assert lib.csa2_index_full_tc(C.byref(kv), C.c_void_p(4104), qbuf, qbuf, 1, 4, 10, 0, 8, None,
                                  qbuf, qbuf, qbuf, 1 << 20, None, None) == 1
    # bad d_idx
    kv2 = pkg.CSA2GlobalKV(256, 256, 256, 256, 1, 100, 96, 1)
    assert lib.csa2_index_reindex(C.byref(kv2), qbuf, qbuf, qbuf, 1, 4, qbuf, 64, 64, qbuf, qbuf,
                                  qbuf, 1 << 20, None, None) == 4
    # attention: H not a multiple of 16, window too small
    swa = pkg.CSA2SWA(256, 256, 1, 128)
    assert lib.csa2_sparse_attn_decode(C.byref(kv), C.byref(swa), qbuf, qbuf, 1, 24, qbuf, 8, 128,
                                       C.c_float(0.04), qbuf, qbuf, None, 0, None, None) == 4
    assert lib.csa2_sparse_attn_decode(C.byref(kv), C.byref(swa), qbuf, qbuf, 4, 64, qbuf, 8, 128,
                                       C.c_float(0.04), qbuf, qbuf, None, 0, None, None) == 2
    # fused append + attention: decode only (Tq = 1), needs the ring and the new row
    assert lib.csa2_sparse_attn_decode_append(C.byref(kv), C.byref(swa), qbuf, qbuf, qbuf, 2, 64,
                                              qbuf, 8, 128, C.c_float(0.04), qbuf, qbuf, None, 0,
                                              None, None) == 4
    assert lib.csa2_sparse_attn_decode_append(C.byref(kv), None, qbuf, qbuf, qbuf, 1, 64, qbuf,
                                              8, 128, C.c_float(0.04), qbuf, qbuf, None, 0, None,
                                              None) == 1
    assert lib.csa2_sparse_attn_decode_append(C.byref(kv), C.byref(swa), C.c_void_p(4100), qbuf,
                                              qbuf, 1, 64, qbuf, 8, 128, C.c_float(0.04), qbuf,
                                              qbuf, None, 0, None, None) == 1
    # the overlapping forms take the same checks: the settled Reindex (bad d_idx), the
    # Reuse attention (H not a multiple of 16; with the fused append: decode only, needs
    # the ring and a 16-byte aligned row; RoPE only with the append)
    assert lib.csa2_index_reindex_settled(C.byref(kv2), qbuf, qbuf, qbuf, 1, 4, qbuf, 64, 64, qbuf,
                                          qbuf, qbuf, 1 << 20, None, None) == 4
    assert lib.csa2_sparse_attn_decode_reuse(C.byref(kv), C.byref(swa), None, qbuf, qbuf, 1, 24, qbuf,
                                             8, 128, C.c_float(0.04), None, qbuf, qbuf, None, None) == 4
    assert lib.csa2_sparse_attn_decode_reuse(C.byref(kv), C.byref(swa), qbuf, qbuf, qbuf, 2, 64, qbuf,
                                             8, 128, C.c_float(0.04), None, qbuf, qbuf, None, None) == 4
    assert lib.csa2_sparse_attn_decode_reuse(C.byref(kv), None, qbuf, qbuf, qbuf, 1, 64, qbuf,
                                             8, 128, C.c_float(0.04), None, qbuf, qbuf, None, None) == 1
    assert lib.csa2_sparse_attn_decode_reuse(C.byref(kv), C.byref(swa), C.c_void_p(4100), qbuf, qbuf, 1,
                                             64, qbuf, 8, 128, C.c_float(0.04), None, qbuf, qbuf, None,
                                             None) == 1
    rope_ok = pkg.CSA2Rope(4096, 8, 0, 4)
    assert lib.csa2_sparse_attn_decode_reuse(C.byref(kv), C.byref(swa), None, qbuf, qbuf, 1, 64, qbuf,
                                             8, 128, C.c_float(0.04), C.byref(rope_ok), qbuf, qbuf, None,
                                             None) == 1
    # their paged forms: a page size that is not a power of two >= 256 is refused first
    pk = pkg.CSA2PagedKV(256, 256, 256, 256, 4096, 1, 4, 100, 8, 128, 1)
    assert lib.csa2_index_reindex_paged_settled(C.byref(pk), qbuf, qbuf, qbuf, 1, 4, qbuf, 64, 64, qbuf,
                                                qbuf, qbuf, 1 << 20, None, None) == 4
    assert lib.csa2_sparse_attn_decode_paged_reuse(C.byref(pk), C.byref(swa), None, qbuf, qbuf, 1, 64, qbuf,
                                                   8, 128, C.c_float(0.04), None, qbuf, qbuf, None, None) == 4
    assert lib.csa2_sparse_attn_decode_paged_reuse(None, C.byref(swa), None, qbuf, qbuf, 1, 64, qbuf,
                                                   8, 128, C.c_float(0.04), None, qbuf, qbuf, None, None) == 1
    # RoPE descriptors: null table, odd start, range past channel 511, no pairs, no rows,
    # misaligned table -- each rejected before any launch, in both _rope calls
    for bad in [(0, 8, 0, 4), (4096, 8, 3, 4), (4096, 8, 500, 8), (4096, 8, 0, 0),
                (4096, 0, 0, 4), (4100, 8, 0, 4)]:
        rope = pkg.CSA2Rope(*bad)
        assert lib.csa2_quantize_append_rope(None, None, None, 0, None, C.byref(swa), qbuf, 1, qbuf,
                                             C.byref(rope), None, None) == 1, bad
        assert lib.csa2_sparse_attn_decode_append_rope(
            C.byref(kv), C.byref(swa), qbuf, qbuf, qbuf, 1, 64, qbuf, 8, 128, C.c_float(0.04),
            C.byref(rope), qbuf, qbuf, None, 0, None, None) == 1, bad
    # append: slot count beyond the cache
    assert lib.csa2_quantize_append(C.byref(kv), qbuf, None, 101, qbuf, None, None, 0, None,
                                    None, None) == 2
    # misaligned cache plane
    kv3 = pkg.CSA2GlobalKV(257, 256, 256, 256, 1, 100, 128, 1)
    assert lib.csa2_index_full(C.byref(kv3), qbuf, qbuf, qbuf, 1, 4, 10, 0, 8, None, qbuf, qbuf,
                               qbuf, 1 << 20, None, None) == 1


def test_plan_layers(pkg):
    plan = pkg.plan_layers(["FUUUXUUUXUUUXUUUXUUU"])
    assert [p.source for p in plan] == [0, 0, 0, 0, 4, 4, 4, 4, 8, 8, 8, 8, 12, 12, 12, 12,
                                        16, 16, 16, 16]
    assert [p.mode for p in plan].count("U") == 15
    plan5 = pkg.plan_layers(["FUUUUU"] * 3 + ["FUUUXUUUXUUUXUUUXUUU"])
    assert len(plan5) == 38
    assert plan5[6].source == 6 and plan5[11].source == 6 and plan5[18].source == 18
    assert plan5[18].group == 3 and plan5[22].source == 22
    with pytest.raises(ValueError):
        pkg.plan_layers(["UF"])
    with pytest.raises(ValueError):
        pkg.plan_layers(["XF"])
