"""csa2_index_full_noalloc: the Full-layer index call for callers that cannot
allocate device memory (a backend running inside a host framework that owns all
device memory, or a loop that cannot take cudaMalloc's device-wide sync).

Called straight through the C ABI; its pool / Top-K / counts must equal those of
csa2_index_full given a caller-owned workspace, bit for bit, on two calls in a
row (the second with a different shape, so stale scratch from the first call
cannot leak into it).  A call needing more than the built-in scratch is refused.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from synth.workloads import WORKLOADS, small_variant

pytestmark = pytest.mark.gpu


def _noalloc_fn(lib):
    fn = lib.csa2_index_full_noalloc
    P, i32 = C.c_void_p, C.c_int32
    fn.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, P, P, P, P, P]
    fn.restype = C.c_int
    return fn


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _run_both(pkg, fn, kv, q_idx, w, q_pos, Tq, H_I, n_max, pool_blocks, top_k, B):
    dev = q_idx.device
    outs = []
    for use_noalloc in (True, False):
        pool = torch.full((B, Tq, max(pool_blocks, 1)), -7, dtype=torch.int32, device=dev)
        topk = torch.full((B, Tq, top_k), -7, dtype=torch.int32, device=dev)
        cnt = torch.full((B, Tq), -7, dtype=torch.int32, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
        if use_noalloc:
            st = fn(C.byref(kv), _ptr(q_idx), _ptr(w), _ptr(q_pos), Tq, H_I, n_max, pool_blocks,
                    top_k, _ptr(pool) if pool_blocks else None, _ptr(topk), _ptr(cnt), _ptr(err),
                    stream)
            assert st == 0, f"csa2_index_full_noalloc returned {st}"
        else:
            ws = torch.empty(pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_FULL, B, Tq, n_max, 0,
                                                     top_k, pool_blocks), dtype=torch.uint8,
                             device=dev)
            pkg.csa2_index_full(kv, q_idx, w, q_pos, Tq, H_I, n_max, pool_blocks, top_k,
                                pool if pool_blocks else None, topk, cnt, ws, err)
        torch.cuda.synchronize()
        assert err.item() == 0
        outs.append((pool.cpu().numpy(), topk.cpu().numpy(), cnt.cpu().numpy()))
    return outs


def test_noalloc_matches_workspace_call_twice():
    import csa2_harness
    import fp4_kv_compressed_b200 as pkg
    assert torch.cuda.is_available()
    fn = _noalloc_fn(pkg.load_library())

    # call 1: hierarchical (pool 2048 x 8 over 20000 entries), 2 requests
    wl = small_variant(WORKLOADS["decoder_group_32k"], B=2, ctx=20000)
    dw = csa2_harness.DeviceWorkload(wl)
    st, inp = dw.stack, dw.inputs
    L = wl.decoder_full_layer
    a, b = _run_both(pkg, fn, st.kv[0].struct, inp["q_idx"][L], inp["w"][L], inp["q_pos"], 1,
                     wl.H_I, 20000, 2048, 512, wl.B)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    assert (a[2] == 512).all()

    # call 2, right after: flat Top-64 of another layer's query at other positions,
    # fewer entries than the first call (the scratch still holds call 1's scores)
    q_pos = torch.tensor([[9000], [4321]], dtype=torch.int32, device="cuda")
    L2 = [lp.layer for lp in st.plan if lp.mode == "X"][0]
    a, b = _run_both(pkg, fn, st.kv[0].struct, inp["q_idx"][L2], inp["w"][L2], q_pos, 1,
                     wl.H_I, 9001, 0, 64, wl.B)
    for x, y in zip(a[1:], b[1:]):
        assert np.array_equal(x, y)
    assert (a[2] == 64).all()

    # beyond the built-in scratch: refused with CSA2_ERR_WORKSPACE, nothing launched
    topk = torch.full((2, 1, 8), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((2, 1), -7, dtype=torch.int32, device="cuda")
    huge = 1 << 30
    st_code = fn(C.byref(st.kv[0].struct), _ptr(inp["q_idx"][L]), _ptr(inp["w"][L]),
                 _ptr(inp["q_pos"]), 1, wl.H_I, huge, 0, 8, None, _ptr(topk), _ptr(cnt), None,
                 C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st_code == 3
    torch.cuda.synchronize()
    assert (cnt == -7).all()
