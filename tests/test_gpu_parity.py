"""GPU parity: every stage of libqsa.so against the CPU oracle, through the
C ABI, on the named workloads at full size (sampled rows where the oracle
would be slow) and on the edge cases of the Ascend operator test list.

Indices (Top-K, expand) are compared bit-exactly on the GPU's own scores;
scores within the dot-product error bound; attention within the max-abs /
mean-abs / rel-L2 tolerances against the FP64 oracle."""
import numpy as np
import pytest
import torch

from indexer_top_sparse_c4_b200 import workloads as wl
from indexer_top_sparse_c4_b200.pipeline import QSAStep
from parity_utils import (ATTN_MAX_ABS, ATTN_MEAN_ABS, ATTN_REL_L2, attn_errors, compact_pages,
                          host, out_as_f64, score_bound)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from indexer_top_sparse_c4_b200 import build
    build.build()


def _rows(T, n=16):
    if T <= n:
        return list(range(T))
    idx = np.unique(np.linspace(0, T - 1, n).astype(int))
    return [int(i) for i in idx]


def _check_step(oracle, w, step, rows=None, check_scores=True):
    """Run the four stages on the GPU and compare each with the oracle fed
    the GPU's previous stage output (scores with their own inputs)."""
    step.run()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    T = w.T
    rows = rows if rows is not None else list(range(T))
    n = {k: host(getattr(w, k)) for k in ("q_idx", "w_idx", "k_idx_pages", "page_table",
                                         "q_req", "q_pos", "q")}
    sel_pos = host(step.sel_pos)
    stride = step.score_stride
    g_scores = host(step.scores)[rows]
    # stage 1: scores within the dot-product error bound
    if check_scores:
        ref, skipped = oracle.index_scores(n["q_idx"][rows], n["w_idx"][rows], n["k_idx_pages"],
                                           n["page_table"], sel_pos[rows], n["q_req"][rows], stride)
        assert skipped == 0
        bound = score_bound(n["q_idx"], n["w_idx"], n["k_idx_pages"], n["page_table"], n["q_req"],
                            sel_pos, rows, stride)
        for i in range(len(rows)):
            c = min(int(sel_pos[rows[i]]) // 4, stride)
            err = np.abs(g_scores[i, :c].astype(np.float64) - ref[i, :c])
            assert np.all(err <= bound[i, :c] + 1e-30), (i, float(err.max()))
    # stage 2: Top-K bit-exact on the GPU's scores
    sel_ref, nsel_ref = oracle.topk_groups(np.ascontiguousarray(g_scores), sel_pos[rows], w.K)
    assert np.array_equal(host(step.n_sel)[rows], nsel_ref)
    assert np.array_equal(host(step.sel)[rows], sel_ref)
    # stage 3: expand bit-exact on the GPU's selection
    cap = None if w.capture_pos is None else host(w.capture_pos)[rows]
    tok_ref, ntok_ref, bad = oracle.expand_select(host(step.sel)[rows], host(step.n_sel)[rows],
                                                  n["q_pos"][rows], w.W, cap)
    assert bad == 0
    assert np.array_equal(host(step.n_tok)[rows], ntok_ref)
    assert np.array_equal(host(step.tok)[rows], tok_ref)
    # stage 4: attention on the GPU's token lists
    tok = host(step.tok)[rows]
    ntok = host(step.n_tok)[rows]
    req = n["q_req"][rows]
    kc, vc, pt = compact_pages(w.k_pages, w.v_pages, w.page_table, tok, ntok, req)
    out_ref, lse_ref, sk = oracle.sparse_attn(n["q"][rows], kc, vc, pt, tok, ntok, w.k_scale,
                                              w.v_scale, q_req=req)
    assert sk == 0
    mx, mean, rel = attn_errors(out_as_f64(step.out)[rows], out_ref)
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel <= ATTN_REL_L2, (mx, mean, rel)
    lse = host(step.lse)[rows].astype(np.float64)
    assert np.abs(lse - lse_ref).max() < 1e-3
    return dict(max_abs=mx, mean_abs=mean, rel_l2=rel)


def test_bound_step_equals_run():
    """QSAStep.bind: the step's calls with their arguments converted once
    give run()'s outputs bit for bit, refilled inputs included."""
    w = wl.b1_16k(device="cuda", B=2, kv_dtype="fp8")
    st = QSAStep(w)
    step = st.bind()
    st.run()
    ref = (st.out.clone(), st.lse.clone(), st.tok.clone())
    st.out.zero_()
    st.tok.zero_()
    step()
    torch.cuda.synchronize()
    assert torch.equal(st.out, ref[0]) and torch.equal(st.lse, ref[1]) and torch.equal(st.tok, ref[2])
    w.q.copy_(torch.flip(w.q, dims=[0]))          # new inputs, same tensors
    step()
    out_b = st.out.clone()
    st.run()
    torch.cuda.synchronize()
    assert torch.equal(out_b, st.out) and int(st.status.item()) == 0


def test_tiny_decode(oracle):
    w = wl.tiny(device="cuda")
    _check_step(oracle, w, QSAStep(w))


def test_b1_decode_16k_bf16(oracle):
    w = wl.b1_16k(device="cuda")
    _check_step(oracle, w, QSAStep(w))


@pytest.mark.parametrize("K", [512, 1024, 2048])
def test_b8_decode_262k_fp8(oracle, K):
    w = wl.b8_262k(K=K, device="cuda")
    _check_step(oracle, w, QSAStep(w), check_scores=(K == 512))


def _single_request_score_bound(q_idx, w_idx, khat, page_table, q_pos, rows, stride, block=256):
    """score_bound() for rows of one request (request 0), in row blocks: the
    request's keys are gathered once and every block is one matmul."""
    from parity_utils import SCORE_REL, values_f64
    P = page_table.shape[1]
    k = np.abs(values_f64(khat[page_table[0]].reshape(P * khat.shape[1], -1)[:stride]))
    for b0 in range(0, len(rows), block):
        rb = rows[b0:b0 + block]
        q = np.abs(values_f64(q_idx[rb]))                             # [n, H, D]
        n, H, D = q.shape
        dots = (q.reshape(n * H, D) @ k.T).reshape(n, H, -1)          # [n, H, stride]
        yield rb, np.einsum("nh,nhg->ng", np.abs(values_f64(w_idx[rb])), dots) * SCORE_REL


def test_prefill_chunk_every_row(oracle):
    """The prefill chunk (8,192 queries): scores of every row within the
    dot-product bound, Top-K and expansion bit-exact on every row (the oracle
    ranks the GPU's own scores), attention on 64 rows, one in each 128-query
    tile of the tensor-core indexer and at a different offset in each."""
    w = wl.prefill_chunk(device="cuda")
    step = QSAStep(w, prefill=True)
    step.run()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    T, stride = w.T, step.score_stride
    n = {k: host(getattr(w, k)) for k in ("q_idx", "w_idx", "k_idx_pages", "page_table", "q_req",
                                         "q_pos", "q")}
    g_scores = host(step.scores)
    c = np.minimum(n["q_pos"].astype(np.int64) // 4, stride)
    # stage 1, every row
    ref, skipped = oracle.index_scores(n["q_idx"], n["w_idx"], n["k_idx_pages"], n["page_table"],
                                       n["q_pos"], n["q_req"], stride)
    assert skipped == 0
    assert np.all(n["q_req"] == 0)
    cols = np.arange(stride)
    for rb, bound in _single_request_score_bound(n["q_idx"], n["w_idx"], n["k_idx_pages"],
                                                  n["page_table"], n["q_pos"], list(range(T)), stride):
        live = cols[None, :] < c[rb][:, None]
        g = g_scores[rb].astype(np.float64)
        assert np.isfinite(g[live]).all(), rb[0]
        err = np.abs(np.where(live, g, 0.0) - np.where(live, ref[rb], 0.0))
        bad = live & ~(err <= bound + 1e-30)
        assert not bad.any(), (rb[0], np.argwhere(bad)[:4])
    del ref
    # stage 2 and 3, every row, bit-exact
    sel_ref, nsel_ref = oracle.topk_groups(g_scores, n["q_pos"], w.K)
    assert np.array_equal(host(step.n_sel), nsel_ref)
    assert np.array_equal(host(step.sel), sel_ref)
    tok_ref, ntok_ref, bad = oracle.expand_select(sel_ref, nsel_ref, n["q_pos"], w.W)
    assert bad == 0
    assert np.array_equal(host(step.n_tok), ntok_ref)
    assert np.array_equal(host(step.tok), tok_ref)
    # stage 4 on one row of every 128-query tile
    rows = [128 * i + (37 * i) % 128 for i in range(T // 128)]
    tok, ntok, req = tok_ref[rows], ntok_ref[rows], n["q_req"][rows]
    kc, vc, pt = compact_pages(w.k_pages, w.v_pages, w.page_table, tok, ntok, req)
    out_ref, lse_ref, sk = oracle.sparse_attn(n["q"][rows], kc, vc, pt, tok, ntok, w.k_scale,
                                              w.v_scale, q_req=req)
    assert sk == 0
    mx, mean, rel = attn_errors(out_as_f64(step.out)[rows], out_ref)
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel <= ATTN_REL_L2, (mx, mean, rel)
    assert np.abs(host(step.lse)[rows].astype(np.float64) - lse_ref).max() < 1e-3


@pytest.mark.parametrize("case", ["ragged_T", "two_requests", "many_runs_odd_stride"])
def test_prefill_indexer_tensor_core_edges(oracle, case):
    """The tcgen05 indexer: a query count that is not a multiple of its
    128-query tiles; request boundaries inside a tile (each run of one
    request's queries gets its own pass, and blocks shared by two runs are
    written row by row); a score stride that is not a multiple of 4 (rows not
    16-byte aligned, so no block store at all)."""
    stride = None
    if case == "ragged_T":
        T, ctx = 1050, 16384
        pos = np.sort(np.random.default_rng(1).integers(12000, ctx, T)).astype(np.int32)
        req = np.zeros(T, np.int32)
        B = 1
    elif case == "two_requests":
        T, ctx = 2048, 8192
        pos = np.concatenate([np.arange(ctx - 1001, ctx), np.arange(ctx - 1047, ctx)]).astype(np.int32)
        req = np.concatenate([np.zeros(1001), np.ones(1047)]).astype(np.int32)
        B = 2
    else:
        T, ctx = 300, 4096
        sizes = [37, 1, 90, 59, 113]   # boundaries at 37, 38, 128, 187 inside the first three tiles
        req = np.concatenate([np.full(n, r % 3) for r, n in enumerate(sizes)]).astype(np.int32)
        pos = np.concatenate([np.sort(np.random.default_rng(n).integers(300, ctx, n)) for n in sizes])
        pos = pos.astype(np.int32)
        B = 3
        stride = ctx // 4 + 3
    w = wl.make(f"tc_{case}", B=B, ctx=ctx, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=256, kv_dtype="bf16",
                q_dtype="bf16", seed=31, device="cuda", q_pos=pos, q_req=req, idx_dtype="bf16")
    step = QSAStep(w, prefill=True, score_stride=stride)
    boundaries = {0, 36, 37, 38, 127, 128, 186, 187, 299, 995, 1000, 1001, 1002, 1023, 1024, 1049}
    rows = sorted(set(_rows(T, 10)) | (boundaries & set(range(T))))
    _check_step(oracle, w, step, rows=rows)


def test_prefill_indexer_bad_request_rows():
    """Rows whose request id is outside the page table get -inf for every
    candidate and raise QSA_DEV_BAD_REQUEST; the rows around them, in the same
    128-query tiles, still score correctly."""
    from indexer_top_sparse_c4_b200 import qsa
    T, ctx = 384, 8192
    pos = np.sort(np.random.default_rng(5).integers(2000, ctx, T)).astype(np.int32)
    w = wl.make("tc_bad_req", B=1, ctx=ctx, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=256, kv_dtype="bf16",
                q_dtype="bf16", seed=9, device="cuda", q_pos=pos, q_req=np.zeros(T, np.int32),
                idx_dtype="bf16")
    w.q_req[200:261] = 7   # the page table has one row
    step = QSAStep(w, prefill=True)
    step.index_scores()
    torch.cuda.synchronize()
    st = int(step.status.item())
    assert st & qsa.QSA_DEV_BAD_REQUEST and not st & qsa.QSA_DEV_TIMEOUT
    scores = host(step.scores)
    for t in range(200, 261):
        assert np.all(np.isneginf(scores[t, : pos[t] // 4]))
    good = [0, 127, 128, 199, 261, 300, 383]
    n = {k: host(getattr(w, k)) for k in ("q_idx", "w_idx", "k_idx_pages", "page_table", "q_req", "q_pos")}
    ref, _ = oracle_scores(n, good, step.score_stride)
    bound = score_bound(n["q_idx"], n["w_idx"], n["k_idx_pages"], n["page_table"], n["q_req"], n["q_pos"],
                        good, step.score_stride)
    for i, t in enumerate(good):
        c = pos[t] // 4
        assert np.all(np.abs(scores[t, :c].astype(np.float64) - ref[i, :c]) <= bound[i, :c] + 1e-30)


def oracle_scores(n, rows, stride):
    import oracle as orc
    return orc.index_scores(n["q_idx"][rows], n["w_idx"][rows], n["k_idx_pages"], n["page_table"],
                            n["q_pos"][rows], n["q_req"][rows], stride)


@pytest.mark.parametrize("case", ["tiny", "b1_16k", "dense_fallback", "prefill_rows", "odd_width"])
def test_topk_expand_matches_separate_calls(case):
    """qsa_topk_expand gives exactly the outputs of qsa_topk_groups followed
    by qsa_expand_select, bit for bit, including the dense fallback (c <= K),
    one-CTA rows (many queries) and a width that is not a multiple of 4."""
    from indexer_top_sparse_c4_b200 import qsa
    if case == "tiny":
        w = wl.tiny(device="cuda")
    elif case == "b1_16k":
        w = wl.b1_16k(device="cuda")
    elif case == "dense_fallback":   # 4,095 candidates, budget 8,192 groups
        w = wl.b1_16k(device="cuda", K=8192)
    else:
        T, ctx = 300, 16384
        pos = np.sort(np.random.default_rng(3).integers(4, ctx, T)).astype(np.int32)
        w = wl.make("rows", B=1, ctx=ctx, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512, kv_dtype="bf16",
                    q_dtype="bf16", seed=4, device="cuda", q_pos=pos, q_req=np.zeros(T, np.int32))
    step = QSAStep(w)
    step.index_scores()
    W = w.W + (1 if case == "odd_width" else 0)
    T, K = w.T, w.K
    outs = []
    for fused in (False, True):
        sel = torch.full((T, K), 7, dtype=torch.int32, device="cuda")
        n_sel = torch.full((T,), 7, dtype=torch.int32, device="cuda")
        tok = torch.full((T, W), 7, dtype=torch.int32, device="cuda")
        n_tok = torch.full((T,), 7, dtype=torch.int32, device="cuda")
        status = torch.zeros((1,), dtype=torch.int32, device="cuda")
        if fused:
            qsa.qsa_topk_expand(step.scores, w.q_pos, K, sel, n_sel, tok, n_tok, dev_status=status)
        else:
            qsa.qsa_topk_groups(step.scores, w.q_pos, K, sel, n_sel, dev_status=status)
            qsa.qsa_expand_select(sel, n_sel, w.q_pos, tok, n_tok, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        outs.append((sel, n_sel, tok, n_tok))
    for x, y in zip(*outs):
        assert torch.equal(x, y)


def _host_prefix_hist(scores, q_pos, stride):
    """Per row: counts of the top 12 bits of the order keys of the candidate
    scores, computed on the host from the GPU's own scores."""
    b = np.ascontiguousarray(scores).view(np.uint32).copy()
    b[b == 0x80000000] = 0
    key = np.where(b & 0x80000000, ~b, b | 0x80000000).astype(np.uint32)
    out = np.zeros((scores.shape[0], 4096), np.int64)
    for t in range(scores.shape[0]):
        c = min(max(int(q_pos[t]), 0) // 4, stride)
        out[t] = np.bincount(key[t, :c] >> 20, minlength=4096)
    return out


def _fake_hist(scores, q_pos, stride, how):
    """A histogram that sums to each row's candidate count but is wrong."""
    h = np.zeros((scores.shape[0], 4096), np.int32)
    true = _host_prefix_hist(scores, q_pos, stride)
    for t in range(scores.shape[0]):
        c = int(true[t].sum())
        nz = np.nonzero(true[t])[0]
        if how == "one_bin":       # every count in the row's highest occupied bin
            h[t, nz.max()] = c
        else:                      # the true counts moved one bin up
            h[t, np.minimum(nz + 1, 4095)] += true[t, nz].astype(np.int32)
    return h


@pytest.mark.parametrize("case", ["b1_16k", "b4_65k_peaked", "b2_262k_peaked", "b2_262k_odd_stride",
                                  "b2_65k_normal_k2048", "ties", "tiny", "dense_fallback", "ragged_rows"])
def test_prefix_hist(case):
    """The scan's prefix histogram equals the one counted on the host from its
    scores; the Top-K (and the fused expansion) given it returns exactly what
    it returns without it, and leaves it zero.  A wrong histogram that still
    sums to the candidate count (every count in one bin; counts moved one bin
    up) changes nothing either: the kernel checks the histogram's bin against
    exact counts before using it."""
    from indexer_top_sparse_c4_b200 import qsa
    if case == "b1_16k":
        w = wl.b1_16k(device="cuda")
    elif case == "b4_65k_peaked":      # clusters of 2 CTAs per row
        w = wl.b8_262k(device="cuda", B=4, ctx=65536)
    elif case in ("b2_262k_peaked", "b2_262k_odd_stride"):     # clusters of 8 CTAs per row
        w = wl.b8_262k(device="cuda", B=2)
    elif case == "b2_65k_normal_k2048":
        w = wl.b8_262k(device="cuda", B=2, ctx=65536, K=2048, dist="normal", kv_dtype="bf16")
    elif case == "ties":   # 16 score levels: the tie bins overflow the candidate lists
        w = wl.b8_262k(device="cuda", B=2, ctx=65536, dist="ties")
    elif case == "tiny":
        w = wl.tiny(device="cuda")
    elif case == "ragged_rows":   # 40 rows of one request, dense and selected rows in one cluster launch
        pos = np.sort(np.random.default_rng(11).integers(4, 65536, 40)).astype(np.int32)
        pos[:3] = [5, 1000, 2050]   # c <= K: the dense rows
        w = wl.make("ragged", B=1, ctx=65536, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512, kv_dtype="fp8",
                    q_dtype="bf16", dist="peaked", seed=12, device="cuda", q_pos=pos,
                    q_req=np.zeros(40, np.int32))
    else:
        w = wl.b1_16k(device="cuda", K=8192)
    # an odd score-row stride takes the Top-K's scalar score loads
    step = QSAStep(w, prefix_hist=True, score_stride=65537 if case == "b2_262k_odd_stride" else None)
    step.index_scores()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    scores = host(step.scores)
    q_pos = host(w.q_pos)
    want = _host_prefix_hist(scores, q_pos, step.score_stride)
    got = host(step.prefix_hist).astype(np.int64)
    assert np.array_equal(got, want)
    saved = step.prefix_hist.clone()
    T, K, W = w.T, w.K, w.W

    def run(hist, fused):
        sel = torch.full((T, K), 7, dtype=torch.int32, device="cuda")
        n_sel = torch.full((T,), 7, dtype=torch.int32, device="cuda")
        tok = torch.full((T, W), 7, dtype=torch.int32, device="cuda")
        n_tok = torch.full((T,), 7, dtype=torch.int32, device="cuda")
        status = torch.zeros((1,), dtype=torch.int32, device="cuda")
        if fused:
            qsa.qsa_topk_expand(step.scores, w.q_pos, K, sel, n_sel, tok, n_tok, dev_status=status,
                                prefix_hist=hist)
        else:
            qsa.qsa_topk_groups(step.scores, w.q_pos, K, sel, n_sel, dev_status=status, prefix_hist=hist)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        return (sel, n_sel, tok, n_tok) if fused else (sel, n_sel)

    for fused in (False, True):
        ref = run(None, fused)
        hists = [saved.clone(),
                 torch.from_numpy(_fake_hist(scores, q_pos, step.score_stride, "one_bin")).cuda(),
                 torch.from_numpy(_fake_hist(scores, q_pos, step.score_stride, "shifted")).cuda()]
        for h in hists:
            got = run(h, fused)
            for x, y in zip(ref, got):
                assert torch.equal(x, y)
            assert int(torch.count_nonzero(h).item()) == 0


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_tensor_parallel_heads(kv):
    """Tensor parallelism over heads needs no library support: each "rank"
    calls the decode attention with its slice of query heads, its KV head's
    cache and the shared selection, and gets its slice of the full output
    and LSE (summation orders differ with the launch shape, so within a
    tolerance far inside the parity bounds)."""
    from indexer_top_sparse_c4_b200 import qsa
    w = wl.b1_16k(device="cuda", kv_dtype=kv, B=2)
    step = QSAStep(w)
    step.run()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    full, full_lse = step.out.float(), step.lse
    G = w.Hq // w.Hkv
    for kvh in range(w.Hkv):
        q = w.q[:, kvh * G:(kvh + 1) * G].contiguous()
        kp = w.k_pages[:, :, kvh:kvh + 1].contiguous()
        vp = w.v_pages[:, :, kvh:kvh + 1].contiguous()
        out = torch.empty((w.T, G, w.D), dtype=step.out.dtype, device="cuda")
        lse = torch.empty((w.T, G), dtype=torch.float32, device="cuda")
        ws_bytes = qsa.qsa_sparse_attn_decode_workspace_size(w.T, G, 1, w.D, w.W, kp.dtype)
        ws = torch.empty((max(ws_bytes, 16),), dtype=torch.uint8, device="cuda")
        status = torch.zeros((1,), dtype=torch.int32, device="cuda")
        qsa.qsa_sparse_attn_decode(q, kp, vp, w.page_table, step.tok, step.n_tok, out, workspace=ws,
                                   k_scale=w.k_scale, v_scale=w.v_scale, q_req=w.q_req, lse=lse,
                                   dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref = full[:, kvh * G:(kvh + 1) * G]
        assert float((out.float() - ref).abs().max()) <= 4e-3
        assert float((lse - full_lse[:, kvh * G:(kvh + 1) * G]).abs().max()) <= 1e-4


GATHER_PLANS = [  # (B, ctx, (Hq, Hkv), K, kv): decode plans of the gather kernel
    (1, 16384, (16, 2), 2048, "bf16"),    # 2 rows x 74 chunks of 112 slots (four two-stage BF16 slots), combine
    (2, 65536, (16, 2), 4096, "fp8"),     # 4 rows x 37 chunks of 448 slots, combine
    (4, 16384, (12, 1), 1024, "fp8"),     # 12 heads per KV head: two warps per slot, 37 chunks per row
    (3, 16384, (6, 1), 512, "bf16"),      # 6 heads per KV head; 33 chunks per row (one tile per slot)
    (40, 8192, (16, 2), 512, "fp8"),      # 80 rows x 3 chunks of 688 (240 CTAs, two waves), combine
    (40, 8192, (16, 2), 128, "fp8"),      # 80 rows of 516 slots: one chunk per row, the output written directly
    (8, 65536, (16, 2), 4096, "fp8"),     # 16 rows x 17 chunks of 976 (the row-index table's 1,024), two waves
]


@pytest.mark.parametrize("case", GATHER_PLANS, ids=lambda c: f"b{c[0]}_c{c[1]}_h{c[2][0]}x{c[2][1]}_k{c[3]}_{c[4]}")
def test_decode_gather_plans(oracle, case):
    """The decode attention's plans: rows split into many chunks merged by
    the combine kernel, one chunk per row written directly, two warps per
    slot, BF16 and FP8 stage sizes, chunks limited by the row-index table;
    every row against the oracle."""
    B, ctx, (Hq, Hkv), K, kv = case
    w = wl.make(f"gather_{B}_{ctx}", B=B, ctx=ctx, Hq=Hq, Hkv=Hkv, D=256, H_I=4, D_I=128, K=K, kv_dtype=kv,
                q_dtype="bf16", dist="peaked", seed=B + K, device="cuda")
    _check_step(oracle, w, QSAStep(w), check_scores=False)


def test_mtp_draft_reuse(oracle):
    w = wl.mtp(device="cuda")
    step = QSAStep(w)
    _check_step(oracle, w, step)
    tok = host(step.tok)
    p0 = int(host(w.capture_pos)[0])
    for t in range(2):   # the group completed since the capture is present
        assert set(range(p0 - 3, p0 + 1)) <= set(tok[t, : host(step.n_tok)[t]].tolist())


@pytest.mark.parametrize("ctx,B,kv", [(16384, 2, "bf16"), (262144, 2, "fp8")])
def test_mtp_draft_loop(oracle, ctx, B, kv):
    """The draft loop with index sharing: each draft step's token list is the
    oracle's expansion of the selection captured at p0 (with the groups
    completed since appended), bit for bit, and its attention matches the
    oracle on that list.  The capture position is the last token of a block,
    so every draft step appends the group completed since."""
    from indexer_top_sparse_c4_b200.pipeline import QSADraftLoop
    p0 = ((ctx - 6) // 4) * 4 + 3
    pos = torch.full((B,), p0, dtype=torch.int32)
    w = wl.make("mtp_capture", B=B, ctx=ctx, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512, kv_dtype=kv,
                q_dtype="bf16", dist="peaked", pages="perm", device="cuda", q_pos=pos,
                q_req=torch.arange(B, dtype=torch.int32))
    loop = QSADraftLoop(w, drafts=2, fused=False)     # the token lists are written: check them
    loop.run()
    fused = QSADraftLoop(w, drafts=2)                 # one call per draft step, same outputs bit for bit
    fused.run()
    torch.cuda.synchronize()
    assert int(loop.status.item()) == 0 and int(fused.status.item()) == 0
    for i in range(loop.drafts):
        assert torch.equal(fused.out[i], loop.out[i]) and torch.equal(fused.lse[i], loop.lse[i])
    n = {k: host(getattr(w, k)) for k in ("page_table", "q_req", "q_pos")}
    sel, n_sel = host(loop.capture.sel), host(loop.capture.n_sel)
    for i in range(loop.drafts):
        tok_ref, ntok_ref, bad = oracle.expand_select(sel, n_sel, host(loop.pos[i]), loop.W, n["q_pos"])
        assert bad == 0
        tok, ntok = host(loop.tok[i]), host(loop.n_tok[i])
        assert np.array_equal(ntok, ntok_ref) and np.array_equal(tok, tok_ref)
        for t in range(B):   # the group completed since the capture is in the list
            assert set(range(p0 - 3, p0 + 1)) <= set(tok[t, :ntok[t]].tolist())
        kc, vc, pt = compact_pages(w.k_pages, w.v_pages, w.page_table, tok, ntok, n["q_req"])
        out_ref, lse_ref, sk = oracle.sparse_attn(host(loop.q[i]), kc, vc, pt, tok, ntok, w.k_scale,
                                                  w.v_scale, q_req=n["q_req"])
        assert sk == 0
        mx, mean, rel = attn_errors(out_as_f64(loop.out[i]), out_ref)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel <= ATTN_REL_L2, (mx, mean, rel)


SWEEP = wl.SWEEP_CASES   # every value of every sweep axis appears at least once


@pytest.mark.parametrize("case", SWEEP, ids=lambda c: f"c{c[0]}_b{c[1]}_h{c[2][0]}x{c[2][1]}_k{c[3]}_{c[4]}_{c[5]}")
def test_sweep(oracle, case):
    ctx, B, heads, K, kv, dist = case
    w = wl.sweep_case(ctx, B, heads, K, kv, dist, device="cuda", seed=ctx + B)
    _check_step(oracle, w, QSAStep(w))


@pytest.mark.parametrize("dist", ["dyadic", "ties"])
def test_chain_indices_bit_exact_on_exact_inputs(oracle, dist):
    """Where every summation order gives the same FP32 score, the whole chain
    (oracle computing its own scores) selects exactly the GPU's groups."""
    w = wl.make(f"exact_{dist}", B=4, ctx=65536, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512,
                kv_dtype="bf16", q_dtype="bf16", dist=dist, seed=21, device="cuda")
    step = QSAStep(w)
    step.run()
    torch.cuda.synchronize()
    n = w.numpy()
    r = oracle.qsa_step(n["q"], n["q_idx"], n["w_idx"], n["k_idx_pages"], n["k_pages"], n["v_pages"],
                        n["page_table"], n["q_pos"], w.K, q_req=n["q_req"])
    c = int(n["q_pos"][0]) // 4
    assert np.array_equal(host(step.scores)[:, :c], r["scores"][:, :c])
    assert np.array_equal(host(step.sel), r["sel"])
    assert np.array_equal(host(step.tok), r["tok"])


def test_chain_on_normal_scores_only_swaps_near_ties(oracle):
    """Raw N(0,1) inputs: scores differ from the oracle by rounding only, so
    any index difference must be a swap at the cut within the score bound."""
    w = wl.make("normal_b8", B=8, ctx=65536, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512,
                kv_dtype="fp8", q_dtype="bf16", dist="normal", seed=22, device="cuda")
    step = QSAStep(w)
    step.run()
    torch.cuda.synchronize()
    n = w.numpy()
    ref, _ = oracle.index_scores(n["q_idx"], n["w_idx"], n["k_idx_pages"], n["page_table"], n["q_pos"],
                                 n["q_req"], step.score_stride)
    sel_ref, _ = oracle.topk_groups(ref, n["q_pos"], w.K)
    bound = score_bound(n["q_idx"], n["w_idx"], n["k_idx_pages"], n["page_table"], n["q_req"],
                        n["q_pos"], range(w.T), step.score_stride)
    gsel = host(step.sel)
    swaps = 0
    for t in range(w.T):
        a, b = set(gsel[t].tolist()), set(sel_ref[t].tolist())
        gpu_only, ref_only = sorted(a - b), sorted(b - a)
        swaps += len(gpu_only)
        if gpu_only:
            # the GPU kept gpu_only over ref_only although the oracle ranks them
            # lower: only possible when each pair's oracle gap is within the two
            # scores' bounds (each GPU score is within its own bound)
            gap = ref[t, ref_only].astype(np.float64).max() - ref[t, gpu_only].astype(np.float64).min()
            assert 0 <= gap <= bound[t, gpu_only].max() + bound[t, ref_only].max(), (t, gap)
    assert swaps <= w.T * 2


# ---- edge cases of the operator test list ------------------------------------------

def _attn_only(oracle, w, tok, n_tok, prefill, sm_scale=0.0, out_dtype=None):
    step = QSAStep(w, prefill=prefill, out_dtype=out_dtype)
    step.tok = torch.as_tensor(tok, dtype=torch.int32, device="cuda").contiguous()
    step.n_tok = torch.as_tensor(n_tok, dtype=torch.int32, device="cuda").contiguous()
    if not prefill:
        from indexer_top_sparse_c4_b200 import qsa
        ws = qsa.qsa_sparse_attn_decode_workspace_size(w.T, w.Hq, w.Hkv, w.D, tok.shape[1],
                                                       w.k_pages.dtype)
        step.ws = torch.empty((max(ws, 16),), dtype=torch.uint8, device="cuda")
    w.W = tok.shape[1]
    step.attention(sm_scale=sm_scale)
    torch.cuda.synchronize()
    n = w.numpy()
    ref, lse, sk = oracle.sparse_attn(n["q"], host(w.k_pages), host(w.v_pages), n["page_table"], tok,
                                      n_tok, w.k_scale, w.v_scale, q_req=n["q_req"], sm_scale=sm_scale)
    return step, ref, lse, sk


@pytest.mark.parametrize("width", [1, 63, 64, 65, 2051])
@pytest.mark.parametrize("prefill", [False, True])
def test_unordered_slots_of_any_width(oracle, width, prefill):
    w = wl.make("slots", B=2, ctx=8192, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512, kv_dtype="bf16",
                q_dtype="bf16", seed=width, device="cuda", q_pos=[8191, 5000], q_req=[0, 1])
    rng = np.random.default_rng(width)
    tok = np.stack([rng.permutation(8192)[:width], rng.permutation(5001)[:width]]).astype(np.int32)
    step, ref, lse, sk = _attn_only(oracle, w, tok, np.array([width, width]), prefill)
    mx, mean, rel = attn_errors(out_as_f64(step.out), ref)
    assert sk == 0 and mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel <= ATTN_REL_L2


@pytest.mark.parametrize("sm_scale", [0.0, 0.03125, 0.2])
def test_default_and_explicit_scale(oracle, sm_scale):
    w = wl.make("scale", B=1, ctx=4096, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512, kv_dtype="fp8",
                q_dtype="bf16", seed=3, device="cuda")
    tok = np.arange(0, 4096, 3, dtype=np.int32)[None]
    step, ref, lse, _ = _attn_only(oracle, w, tok, np.array([tok.shape[1]]), False, sm_scale)
    mx, mean, rel = attn_errors(out_as_f64(step.out), ref)
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel <= ATTN_REL_L2
    assert np.abs(host(step.lse) - lse).max() < 1e-3


@pytest.mark.parametrize("prefill", [False, True])
def test_masked_and_zero_rows_are_exact_zero(oracle, prefill):
    w = wl.make("empty", B=3, ctx=1024, Hq=6, Hkv=1, D=256, H_I=4, D_I=128, K=64, kv_dtype="bf16",
                q_dtype="bf16", seed=4, device="cuda", q_pos=[1023, 1023, 1023], q_req=[0, 1, 2])
    tok = np.full((3, 64), -1, np.int32)
    tok[2, :5] = [1, 2, 3, 700, 1023]
    n_tok = np.array([64, 0, 5])          # all -1 / width 0 / normal
    step, ref, lse, _ = _attn_only(oracle, w, tok, n_tok, prefill)
    out = out_as_f64(step.out)
    assert np.all(out[:2] == 0) and np.all(host(step.lse)[:2] == -np.inf)
    assert attn_errors(out[2:], ref[2:])[0] <= ATTN_MAX_ABS


@pytest.mark.parametrize("rem", [0, 1, 2, 3])
def test_causal_tail_remainders(oracle, rem):
    """p % 4 = 0..3: the current block holds 1..4 tokens and always the query."""
    p = 4 * 1000 + rem
    w = wl.make("tail", B=1, ctx=p + 1, Hq=12, Hkv=1, D=256, H_I=4, D_I=128, K=128, kv_dtype="bf16",
                q_dtype="bf16", seed=rem, device="cuda")
    step = QSAStep(w)
    _check_step(oracle, w, step)
    row = host(step.tok)[0, : host(step.n_tok)[0]]
    assert row[-1] == p and list(row[-(rem + 1):]) == list(range(4 * 1000, p + 1))


def test_selection_width_zero_before_first_group(oracle):
    """p < 4: no complete group, n_sel = 0, only the current block is attended."""
    w = wl.make("w0", B=3, ctx=64, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=8, kv_dtype="bf16",
                q_dtype="bf16", seed=5, device="cuda", q_pos=[0, 2, 3], q_req=[0, 1, 2])
    step = QSAStep(w)
    _check_step(oracle, w, step)
    assert host(step.n_sel).tolist() == [0, 0, 0]
    assert host(step.n_tok).tolist() == [1, 3, 4]


def test_two_requests_sharing_prefix_pages(oracle):
    w = wl.make("shared", B=2, ctx=8192, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=256, kv_dtype="fp8",
                q_dtype="bf16", seed=6, device="cuda")
    w.page_table[1, :64] = w.page_table[0, :64]     # first 4,096 tokens shared
    w.q_idx[1] = w.q_idx[0]
    w.w_idx[1] = w.w_idx[0]
    step = QSAStep(w)
    _check_step(oracle, w, step)


def test_cache_content_reuse_is_deterministic():
    w = wl.b1_16k(device="cuda", seed=7)
    step = QSAStep(w)
    step.run()
    a = [t.clone() for t in (step.scores, step.sel, step.tok, step.out, step.lse)]
    step.run()
    torch.cuda.synchronize()
    for x, y in zip(a, (step.scores, step.sel, step.tok, step.out, step.lse)):
        assert torch.equal(x, y)


@pytest.mark.parametrize("heads", [(16, 2), (24, 2), (12, 1), (6, 1), (3, 1)])
@pytest.mark.parametrize("T", [1, 257])
def test_local_head_shapes_prefill_rows(oracle, heads, T):
    Hq, Hkv = heads
    ctx = 16384
    pos = np.sort(np.random.default_rng(T).integers(8000, ctx, T)).astype(np.int32)
    w = wl.make("heads", B=1, ctx=ctx, Hq=Hq, Hkv=Hkv, D=256, H_I=4, D_I=128, K=512, kv_dtype="bf16",
                q_dtype="bf16", seed=Hq * T, device="cuda", q_pos=pos, q_req=np.zeros(T, np.int32))
    step = QSAStep(w, prefill=True)
    _check_step(oracle, w, step, rows=_rows(T, 6))


def test_bad_page_id_is_flagged_not_trapped():
    from indexer_top_sparse_c4_b200 import qsa
    w = wl.make("bad", B=1, ctx=4096, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=64, kv_dtype="bf16",
                q_dtype="bf16", seed=8, device="cuda")
    w.page_table[0, 5] = 10 ** 6
    step = QSAStep(w)
    step.run()
    torch.cuda.synchronize()
    st = int(step.status.item())
    assert st & qsa.QSA_DEV_BAD_PAGE
    assert torch.isfinite(step.out.float()).all()
    # the same word through the C ABI's status query, which also clears it
    code, bits = qsa.qsa_get_device_status(step.status, clear=True)
    assert code == qsa.QSA_ERR_DEVICE_INDEX and bits == st
    assert "page" in qsa.qsa_last_error_string()
    assert qsa.qsa_get_device_status(step.status) == (qsa.QSA_OK, 0)
    assert int(step.status.item()) == 0


def test_non_contiguous_input_is_refused():
    w = wl.tiny(device="cuda")
    step = QSAStep(w)
    w.q_idx = w.q_idx.transpose(1, 2)
    with pytest.raises(ValueError, match="contiguous"):
        step.index_scores()
