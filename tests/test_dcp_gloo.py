"""Sequence-sharded decode on CPU ranks (gloo, world size 2 and 4): every rank
runs the oracle on its own slice of the page table -- its groups' scores,
its exact local top-K as (score, global id) records -- the records are
all-gathered, merged into the global top-K, every rank attends over its part
of the selection, the partial (out, lse) are all-gathered and merged by LSE.
The result must be the unsharded oracle's: the same selection, bit for bit,
and the same output up to FP64 rounding.  This checks the decomposition and
the host logic of the sharded path (shard bounds, gathers) without a GPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _merge_topk(score, ids, K):
    """Plain merge of the gathered records [R, T, K]: per row, the K best by
    (score descending, id ascending), returned ascending by id."""
    R, T, _ = ids.shape
    sel = np.full((T, K), -1, np.int32)
    n_sel = np.zeros((T,), np.int32)
    for t in range(T):
        s, i = score[:, t].reshape(-1), ids[:, t].reshape(-1)
        ok = i >= 0
        s, i = s[ok].astype(np.float64), i[ok]
        s[s == 0] = 0.0
        order = np.lexsort((i, -s))[:K]
        keep = np.sort(i[order])
        sel[t, :len(keep)] = keep
        n_sel[t] = len(keep)
    return sel, n_sel


def _rank_main(rank, world, port, q, case):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from indexer_top_sparse_c4_b200 import dcp
        from indexer_top_sparse_c4_b200 import workloads as wl
        dist_name, K = case
        w = wl.make("dcp", B=2, ctx=4096 + 7, Hq=4, Hkv=1, D=64, H_I=2, D_I=32, K=K, kv_dtype="f32",
                    q_dtype="f32", dist=dist_name, pages="perm", seed=5)
        w.q_pos[1] = 2050                                  # the second request queries mid-context
        n = w.numpy()
        T, P = w.T, n["page_table"].shape[1]
        lo, hi = dcp.shard_bounds(P, world)[rank]
        g_lo, g_hi = lo * 16, hi * 16
        pt = np.ascontiguousarray(n["page_table"][:, lo:hi])
        c = n["q_pos"] // 4
        q_local = (4 * np.clip(c - g_lo, 0, g_hi - g_lo)).astype(np.int32)
        stride = max(1, g_hi - g_lo)
        scores, _ = oracle.index_scores(n["q_idx"], n["w_idx"], n["k_idx_pages"], pt, q_local, n["q_req"], stride)
        sel_r, nsel_r = oracle.topk_groups(scores, q_local, K)
        cid = np.full((T, K), -1, np.int32)
        csc = np.full((T, K), -np.inf, np.float32)
        for t in range(T):
            m = nsel_r[t]
            cid[t, :m] = sel_r[t, :m] + g_lo
            csc[t, :m] = scores[t, sel_r[t, :m]]
        ids = dcp.gather(torch.from_numpy(cid)).numpy()
        sc = dcp.gather(torch.from_numpy(csc)).numpy()
        sel, n_sel = _merge_topk(sc, ids, K)
        # this shard's part of the selection, as shard-local token ids
        W = 4 * K + 4
        tok = np.full((T, W), -1, np.int32)
        ntok = np.zeros((T,), np.int32)
        for t in range(T):
            row = [4 * (g - g_lo) + j for g in sel[t, :n_sel[t]] if g_lo <= g < g_hi for j in range(4)]
            if g_lo <= c[t] < g_hi:
                row += list(range(4 * (c[t] - g_lo), n["q_pos"][t] - 4 * g_lo + 1))
            tok[t, :len(row)] = row
            ntok[t] = len(row)
        o_r, lse_r, sk = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], pt, tok, ntok, q_req=n["q_req"])
        assert sk == 0
        o_all = dcp.gather(torch.from_numpy(o_r)).numpy()
        lse_all = dcp.gather(torch.from_numpy(lse_r)).numpy()
        LSE = np.logaddexp.reduce(lse_all, axis=0)
        wts = np.where(np.isneginf(lse_all), 0.0, np.exp(lse_all - LSE))
        out = np.einsum("rth,rthd->thd", wts, o_all)
        ref = oracle.qsa_step(n["q"], n["q_idx"], n["w_idx"], n["k_idx_pages"], n["k_pages"], n["v_pages"],
                              n["page_table"], n["q_pos"], K, q_req=n["q_req"])
        q.put((rank, np.array_equal(sel, ref["sel"]), np.array_equal(n_sel, ref["n_sel"]),
               float(np.abs(out - ref["out"]).max()), float(np.abs(LSE - ref["lse"]).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("case", [("normal", 48), ("ties", 48), ("normal", 2000)],
                         ids=["normal_k48", "ties_k48", "dense_k2000"])
def test_sharded_decode_equals_unsharded(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, case)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, sel_ok, nsel_ok, err, lse_err in res:
        assert sel_ok and nsel_ok, rank
        assert err < 1e-9 and lse_err < 1e-9, (rank, err, lse_err)


def test_shard_bounds_cover_the_pages_once():
    import sys
    sys.path.insert(0, ROOT)
    from indexer_top_sparse_c4_b200.dcp import shard_bounds
    for P in (1, 7, 64, 4096, 4097):
        for R in (1, 2, 3, 4, 8):
            b = shard_bounds(P, R)
            assert len(b) == R and b[0][0] == 0 and b[-1][1] == P
            assert all(b[i][1] == b[i + 1][0] for i in range(R - 1))
            sizes = [hi - lo for lo, hi in b]
            assert max(sizes) - min(sizes) <= 1
