"""Host logic of the context-parallel path on two gloo ranks (CPU).

fp4_kv_compressed_b200.context_parallel orders the calls of one rank and does its two
all-gathers; the kernels themselves are checked on the GPU (test_gpu_cp.py).  Here the
compute calls go to a numpy stand-in with the same contracts (candidate keys, exact
merge in (key desc, id asc) order, normalised partial softmax, log-sum-exp combine), so
that the slicing, the all-gather order, the slice-local ids, the window owner and the
combine are exercised through real torch.distributed collectives.  Each rank's result
must equal the unsharded run of the same stand-in."""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

B, TQ, H, D = 2, 1, 4, 512
N, POOL, TOPK, WIN = 1000, 32, 24, 8
SCALE = 0.05


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _key(x: np.ndarray) -> np.ndarray:
    """Order key of fp32 scores: larger score, larger key; never 0."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return np.where(u & 0x80000000, (~u) & 0xFFFFFFFF, u | 0x80000000)


class FakeKV:
    """The slice [lo, lo + cap) of every request: scores and value rows by global id."""

    def __init__(self, scores, values, lo, cap):
        self.scores, self.values, self.lo, self.cap, self.ratio = scores, values, lo, cap, 1


class NumpyBackend:
    @staticmethod
    def index_full_slice(kv, lo, q_idx, w, q_pos, Tq, H_I, n_max, P, K, pool_keys, topk_keys,
                         ws, err, stream):
        for b in range(q_pos.shape[0]):
            n = max(0, min(kv.cap, int(q_pos[b, 0]) + 1 - lo))
            s = kv.scores[b, lo:lo + n]
            ids = np.arange(lo, lo + n)
            order = np.lexsort((ids, -s))[:K]
            sel = np.sort(ids[order])
            keys = (_key(kv.scores[b, sel]) << 32) | (~sel.astype(np.uint64) & 0xFFFFFFFF)
            topk_keys[b, 0, :len(sel)] = torch.from_numpy(keys.view(np.int64))
            nb = -(-n // 8)
            bm = np.array([kv.scores[b, lo + 8 * i:lo + min(n, 8 * i + 8)].max() for i in range(nb)])
            bids = np.arange(nb) + lo // 8
            border = np.sort(bids[np.lexsort((bids, -bm))[:P]])
            bkeys = (_key(bm[border - lo // 8]) << 32) | (~border.astype(np.uint64) & 0xFFFFFFFF)
            pool_keys[b, 0, :len(border)] = torch.from_numpy(bkeys.view(np.int64))

    @staticmethod
    def index_merge(lists, BT, n_lists, n, k, lo, hi, ids_out, count_out, local_out, stream):
        L = lists.numpy().view(np.uint64).reshape(n_lists, BT, n)
        for q in range(BT):
            c = L[:, q, :].ravel()
            c = c[c != 0]
            ids = (~c & 0xFFFFFFFF).astype(np.int64)
            top = np.sort(ids[np.lexsort((ids, -(c >> 32).astype(np.int64)))[:k]])
            row = np.full(k, -1, np.int32)
            row[:len(top)] = top
            ids_out.view(-1, k)[q] = torch.from_numpy(row)
            if count_out is not None:
                count_out.view(-1)[q] = len(top)
            loc = np.where((row >= lo) & (row < hi), row - lo, -1).astype(np.int32)
            local_out.view(-1, k)[q] = torch.from_numpy(loc)

    @staticmethod
    def attention(kv, swa, q, q_pos, Tq, H_, topk_local, top_k, swa_len, scale, out, lse, err,
                  stream):
        for b in range(q.shape[0]):
            ids = [kv.lo + int(e) for e in topk_local[b, 0] if e >= 0]
            vals = [kv.values[b, i] for i in ids]
            if swa is not None:
                t = int(q_pos[b, 0])
                vals += [swa[b, p] for p in range(max(0, t - swa_len + 1), t + 1)]
            if not vals:
                continue
            V = np.stack(vals).astype(np.float64)
            lg = scale * (q[b, 0].numpy().astype(np.float64) @ V.T)
            m = lg.max(-1, keepdims=True)
            p = np.exp(lg - m)
            out[b, 0] = torch.from_numpy(p @ V / p.sum(-1, keepdims=True)).float()
            lse[b, 0] = torch.from_numpy(m[:, 0] + np.log(p.sum(-1))).float()

    @staticmethod
    def combine(o_parts, l_parts, n_parts, rows, out, lse, stream):
        lp = l_parts.double()
        m = lp.max(0).values
        wgt = torch.where(torch.isinf(lp), torch.zeros_like(lp), torch.exp(lp - m))
        s = wgt.sum(0)
        out.copy_((wgt[..., None] * o_parts.double()).sum(0) / s[..., None])
        lse.copy_(m + torch.log(s))


def _inputs():
    g = np.random.default_rng(5)
    scores = g.standard_normal((B, N)).astype(np.float32)
    scores[:, 100:110] = 1.5                               # exact ties across a slice bound
    values = g.standard_normal((B, N, D)).astype(np.float32)
    swa = g.standard_normal((B, N, D)).astype(np.float32)
    q = torch.from_numpy(g.standard_normal((B, TQ, H, D)).astype(np.float32))
    q_pos = torch.tensor([[N - 1], [555]], dtype=torch.int32)
    return scores, values, swa, q, q_pos


def _run(shard, swa, q, q_pos):
    res = shard.full_select(None, None, q_pos, TQ, 4, POOL, TOPK, None)
    out, lse = shard.attend(swa, q, q_pos, TQ, H, res.topk_local, TOPK, WIN, SCALE)
    return res.pool.numpy(), res.topk.numpy(), res.count.numpy(), out.numpy(), lse.numpy()


def _rank_main(rank, world, port, q_out):
    import datetime
    import torch.distributed as dist
    from fp4_kv_compressed_b200.context_parallel import ContextShard, dist_gather, slice_bounds
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        scores, values, swa, q, q_pos = _inputs()
        lo, hi = slice_bounds(N, world)[rank]
        shard = ContextShard(FakeKV(scores, values, lo, hi - lo), lo, hi, rank, world,
                             window=rank == world - 1, gather=dist_gather, backend=NumpyBackend)
        q_out.put((rank, _run(shard, swa, q, q_pos)))
    finally:
        dist.destroy_process_group()


def test_slice_bounds():
    from fp4_kv_compressed_b200.context_parallel import slice_bounds
    for n, w in ((1000, 2), (1000, 3), (64, 4), (0, 2), (131072, 8), (20001, 7)):
        b = slice_bounds(n, w)
        assert b[0][0] == 0 and b[-1][1] == n and len(b) == w
        for (lo, hi), (lo2, _) in zip(b, b[1:]):
            assert hi == lo2 and lo % 64 == 0
        assert all(lo <= hi for lo, hi in b)


def test_two_gloo_ranks_match_unsharded():
    from fp4_kv_compressed_b200.context_parallel import ContextShard
    scores, values, swa, q, q_pos = _inputs()
    one = ContextShard(FakeKV(scores, values, 0, N), 0, N, 0, 1, window=True,
                       gather=lambda t: t[None], backend=NumpyBackend)
    ref = _run(one, swa, q, q_pos)
    world = 2
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, qq)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(qq.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        pool, topk, count, out, lse = res[r]
        assert np.array_equal(pool, ref[0]) and np.array_equal(topk, ref[1])
        assert np.array_equal(count, ref[2])
        assert np.allclose(out, ref[3], rtol=1e-5, atol=1e-6)
        assert np.allclose(lse, ref[4], rtol=1e-6, atol=1e-6)
