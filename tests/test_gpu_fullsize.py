"""GPU parity at the workloads' full sizes, in the benchmark's launch configuration
(one DecodeStack step through the library, whole batch), checked on sampled
requests, layers and query tokens that the oracle recomputes one by one:

* the sampled requests' whole indexer-K planes (codes and scales) bit for bit;
* the main-KV entries every selector layer picked, bit for bit;
* every Full / Reindex layer's pool, Top-K and count bit for bit;
* attention of sampled layers within the 2e-3 norm-wise bound.

Queries are independent given the caches, so a query-token subset of a prefill
chunk is checked exactly like a whole batch.
"""
import numpy as np
import pytest
import torch

from oracle import workload_ref as R
from synth.workloads import WORKLOADS

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

ATTN_TOL = 2e-3
LSE_TOL = 1e-3


def _sampled_check(name, requests, layers, qsel=None):
    import csa2_harness
    wl = WORKLOADS[name]
    dw = csa2_harness.DeviceWorkload(wl)
    dw.step()
    torch.cuda.synchronize()
    st = dw.stack
    assert st.dev_err.item() == 0
    plan = R.reuse_sources(wl)
    sel = slice(None) if qsel is None else torch.as_tensor(qsel)
    for b in requests:
        topk_gpu = {l: t[b][sel].cpu().numpy() for l, t in st.topk.items()}
        count_gpu = {l: c[b][sel].cpu().numpy() for l, c in st.count.items()}
        rows = {g: [] for g in range(len(wl.groups))}
        for layer, t in topk_gpu.items():
            rows[plan[layer][0]].append(t.ravel())
        rows = {g: np.concatenate(v) if v else np.zeros(0, np.int64) for g, v in rows.items()}
        caches = R.request_caches(wl, b, main_rows=rows)
        for g, c in enumerate(caches):
            N = c["N"]
            kv = st.kv[g]
            assert np.array_equal(kv.idx_codes[b, :N].cpu().numpy(), c["idx_codes"]), f"g{g} idx"
            assert np.array_equal(kv.idx_scale[b, :N].cpu().numpy().view(np.uint32),
                                  c["idx_scale"].view(np.uint32)), f"g{g} idx scale"
            r = torch.as_tensor(c["rows"], dtype=torch.int64)
            assert np.array_equal(kv.codes[b][r.to(kv.codes.device)].cpu().numpy(),
                                  c["codes"][c["rows"]]), f"g{g} codes"
            assert np.array_equal(kv.scales[b][r.to(kv.scales.device)].cpu().numpy(),
                                  c["scales"][c["rows"]]), f"g{g} scales"
        ref = R.index_layers(wl, b, caches, qsel=qsel)
        for layer, t in ref["topk"].items():
            assert np.array_equal(count_gpu[layer], ref["count"][layer]), f"b{b} L{layer} count"
            assert np.array_equal(topk_gpu[layer], t), f"b{b} L{layer} Top-K"
        for g, p in ref["pool"].items():
            assert np.array_equal(st.pool[g][b][sel].cpu().numpy(), p), f"b{b} g{g} pool"
        for layer in layers:
            src = plan[layer][2]
            o_ref, l_ref = R.attention_layer(wl, b, layer, caches, ref["topk"][src], qsel=qsel)
            o = st.out[layer][b][sel].cpu().numpy()
            l = st.lse[layer][b][sel].cpu().numpy()
            err = R.rel_err_rows(o, o_ref)
            print(f"{name} b{b} L{layer}: norm-wise row error {err.max():.2e}, elementwise "
                  f"(|o_ref| >= row RMS) {R.rel_err_elems(o, o_ref):.2e}")
            assert err.max() <= ATTN_TOL, f"b{b} L{layer} max row error {err.max():.3e}"
            assert np.abs(l - l_ref).max() <= LSE_TOL, f"b{b} L{layer} lse"
    del dw
    torch.cuda.empty_cache()


def test_decode_128k_full_size():
    """Batch 64 at context 131072, the 20-layer decoder stack: requests 0 and 63, the
    Full layer, two Reindex layers and a Reuse layer."""
    _sampled_check("decode_128k", [0, 63], layers=[0, 4, 12, 19])


def test_decoder_group_32k_full_size():
    """Batch 8 at context 32768 with planted positions: every layer of requests 0 and 7."""
    _sampled_check("decoder_group_32k", [0, 7], layers=list(range(20)))


def test_prefill_chunk_full_size():
    """2048 causal queries after a 65536-token prefix (ratio 2, flat): 6 sampled query
    tokens, from the first to the last of the chunk, every layer."""
    _sampled_check("prefill_chunk_enc", [0], layers=list(range(6)),
                   qsel=np.array([0, 1, 255, 1024, 2046, 2047]))


def test_decode_1m_full_size():
    """Batch 4 at context 1048576, 3 flat encoder groups + the decoder group: the last
    request, each group's Full layer and one Reuse / Reindex layer."""
    _sampled_check("decode_1m", [3], layers=[0, 5, 6, 18, 19, 23, 37])
