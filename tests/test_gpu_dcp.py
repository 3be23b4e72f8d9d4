"""Sequence-sharded decode on one GPU: R shards run in turn through the
library over slices of the page table; their candidate records and partial
attentions are merged by the library's merge kernels.  The selection must
equal the unsharded path's bit for bit (same scores: each group's score does
not depend on the shard), the oracle's Top-K of those scores, and the output
must match the oracle within the attention tolerances."""
import numpy as np
import pytest
import torch

from indexer_top_sparse_c4_b200 import workloads as wl
from indexer_top_sparse_c4_b200.pipeline import QSAStep
from parity_utils import ATTN_MAX_ABS, ATTN_MEAN_ABS, ATTN_REL_L2, attn_errors, compact_pages, host, out_as_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from indexer_top_sparse_c4_b200 import build
    build.build()


CASES = [  # (B, ctx, K, kv, dist, shards)
    (8, 65536, 512, "fp8", "peaked", 2),
    (8, 65536, 2048, "fp8", "peaked", 4),
    (2, 262144, 1024, "fp8", "peaked", 3),
    (4, 16384, 512, "bf16", "ties", 4),
    (2, 8192 + 37, 4096, "bf16", "normal", 3),   # c <= K on some shards: dense rows
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"b{c[0]}_c{c[1]}_k{c[2]}_{c[3]}_{c[4]}_r{c[5]}")
def test_sharded_decode_matches_unsharded(oracle, case):
    from indexer_top_sparse_c4_b200.dcp import QSADcpDecode
    B, ctx, K, kv, dist, R = case
    w = wl.make("dcp", B=B, ctx=ctx, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=K, kv_dtype=kv, q_dtype="bf16",
                dist=dist, pages="perm", seed=B + R, device="cuda")
    if B > 1:
        w.q_pos[1] = ctx // 2 + 5                # a query in mid-context: its current block sits on an inner shard
    full = QSAStep(w)
    full.run()
    d = QSADcpDecode(w, R)
    d.run()
    torch.cuda.synchronize()
    assert int(full.status.item()) == 0 and int(d.status.item()) == 0
    assert torch.equal(d.n_sel, full.n_sel)
    assert torch.equal(d.sel, full.sel)
    n = {k: host(getattr(w, k)) for k in ("q", "page_table", "q_req", "q_pos")}
    sel_ref, nsel_ref = oracle.topk_groups(host(full.scores), n["q_pos"], K)
    assert np.array_equal(host(d.sel), sel_ref) and np.array_equal(host(d.n_sel), nsel_ref)
    # every shard's token list is its part of the full list, shifted to local ids
    ft, fn = host(full.tok), host(full.n_tok)
    parts = {r: (host(d.sh[r]["tok"]), host(d.sh[r]["n_tok"])) for r in d.mine}
    for t in range(w.T):
        merged = []
        for r in range(R):
            tok, nt = parts[r]
            merged += [x + 64 * d.bounds[r][0] for x in tok[t, :nt[t]]]
        assert merged == list(ft[t, :fn[t]]), t
    # the merged output against the oracle on the full list
    kc, vc, pt = compact_pages(w.k_pages, w.v_pages, w.page_table, ft, fn, n["q_req"])
    ref, lse_ref, sk = oracle.sparse_attn(n["q"], kc, vc, pt, ft, fn, w.k_scale, w.v_scale, q_req=n["q_req"])
    assert sk == 0
    mx, mean, rel = attn_errors(out_as_f64(d.out), ref)
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel <= ATTN_REL_L2, (mx, mean, rel)
    assert np.abs(host(d.lse).astype(np.float64) - lse_ref).max() < 1e-3


def test_merge_attn_of_empty_shards_is_zero():
    """Rows where every shard attended nothing give 0 and -inf; a shard with
    nothing contributes nothing to the others."""
    from indexer_top_sparse_c4_b200 import qsa
    R, T, Hq, D = 3, 2, 4, 64
    o = torch.randn((R, T, Hq, D), device="cuda")
    lse = torch.full((R, T, Hq), float("-inf"), device="cuda")
    lse[1, 1] = 0.5                                   # row 1: only shard 1 has tokens
    out = torch.empty((T, Hq, D), dtype=torch.float32, device="cuda")
    lo = torch.empty((T, Hq), dtype=torch.float32, device="cuda")
    qsa.qsa_dcp_merge_attn(o, lse, out, lo)
    torch.cuda.synchronize()
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lo[0]))
    assert torch.allclose(out[1], o[1, 1], atol=1e-6) and torch.allclose(lo[1], lse[1, 1])


def test_merge_topk_ties_go_to_the_lower_id():
    """Records with equal scores across shards: the lower global ids win,
    output ascending, padding records ignored."""
    from indexer_top_sparse_c4_b200 import qsa
    R, T, K = 2, 1, 4
    score = torch.tensor([[[1.0, 2.0, 2.0, float("-inf")]], [[2.0, 2.0, 0.5, 3.0]]], device="cuda")
    ids = torch.tensor([[[3, 5, 9, -1]], [[20, 21, 30, 40]]], dtype=torch.int32, device="cuda")
    sel = torch.empty((T, K), dtype=torch.int32, device="cuda")
    n_sel = torch.empty((T,), dtype=torch.int32, device="cuda")
    qsa.qsa_dcp_merge_topk(score, ids, sel, n_sel)
    torch.cuda.synchronize()
    # 3.0 (40), then the 2.0 ties 5, 9, 20, 21 -> the lower three: 5, 9, 20
    assert n_sel.tolist() == [4] and sel.tolist() == [[5, 9, 20, 40]]
