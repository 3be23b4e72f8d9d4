"""The guess-verify-refine Top-K (self-sampling): the same selection as the
exact radix Top-K and the oracle, bit for bit, on the GPU's own scores, for
every budget it serves and every score distribution; the path record shows
that the self-sampled guess is what selects on ordinary rows, and that rows
where guessing cannot work (thousands of equal scores) take the whole-row
select."""
import numpy as np
import pytest
import torch

from indexer_top_sparse_c4_b200 import workloads as wl
from indexer_top_sparse_c4_b200.pipeline import QSAStep
from parity_utils import host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from indexer_top_sparse_c4_b200 import build, qsa
    build.build()
    return qsa


def _gvr(q, scores, q_pos, K):
    T = scores.shape[0]
    sel = torch.full((T, K), 7, dtype=torch.int32, device="cuda")
    n_sel = torch.full((T,), 7, dtype=torch.int32, device="cuda")
    path = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    q.qsa_topk_groups_gvr(scores, q_pos, K, sel, n_sel, path=path)
    torch.cuda.synchronize()
    return sel, n_sel, path


def _radix(q, scores, q_pos, K):
    T = scores.shape[0]
    sel = torch.empty((T, K), dtype=torch.int32, device="cuda")
    n_sel = torch.empty((T,), dtype=torch.int32, device="cuda")
    q.qsa_topk_groups(scores, q_pos, K, sel, n_sel)
    torch.cuda.synchronize()
    return sel, n_sel


@pytest.mark.parametrize("K", [512, 1024, 2048])
@pytest.mark.parametrize("dist", ["peaked", "normal", "ties"])
def test_gvr_equals_radix_and_oracle_on_decode_rows(q, oracle, K, dist):
    w = wl.b8_262k(K=K, device="cuda", dist=dist, B=4, ctx=65536 if dist == "ties" else 262144)
    st = QSAStep(w, prefix_hist=False)
    st.index_scores()
    sel, n_sel, path = _gvr(q, st.scores, w.q_pos, K)
    rs, rn = _radix(q, st.scores, w.q_pos, K)
    assert torch.equal(sel, rs) and torch.equal(n_sel, rn)
    ref, nref = oracle.topk_groups(host(st.scores), host(w.q_pos), K)
    assert np.array_equal(host(sel), ref) and np.array_equal(host(n_sel), nref)
    p = host(path)
    if dist == "ties":   # 16 score levels: the guess may land on a crowded level
        assert set(p.tolist()) <= {1, 2, 3}
    else:
        assert np.all(p == 1), p                     # the first self-sampled guess verifies


def test_gvr_rows_of_every_length(q, oracle):
    """Prefill-like rows: dense rows (c <= K), rows just above K, long rows,
    an odd score stride; all against the radix Top-K and the oracle."""
    T, ctx, K = 300, 16384, 512
    pos = np.sort(np.random.default_rng(3).integers(4, ctx, T)).astype(np.int32)
    pos[:4] = [5, 2047, 2051, 2052]
    w = wl.make("rows", B=1, ctx=ctx, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=K, kv_dtype="bf16", q_dtype="bf16",
                seed=4, device="cuda", q_pos=pos, q_req=np.zeros(T, np.int32))
    st = QSAStep(w, score_stride=ctx // 4 + 1)
    st.index_scores()
    sel, n_sel, path = _gvr(q, st.scores, w.q_pos, K)
    rs, rn = _radix(q, st.scores, w.q_pos, K)
    assert torch.equal(sel, rs) and torch.equal(n_sel, rn)
    ref, nref = oracle.topk_groups(host(st.scores), host(w.q_pos), K)
    assert np.array_equal(host(sel), ref)
    p = host(path)
    c = pos // 4
    assert np.all(p[c <= K] == 0) and np.all(p[c > K] >= 1)


def test_gvr_falls_back_on_equal_scores(q, oracle):
    """Every candidate with the same score: no threshold can split them, the
    row takes the whole-row select, and the lowest ids win."""
    T, c, K = 2, 65535, 1024
    scores = torch.zeros((T, c + 1), dtype=torch.float32, device="cuda")
    scores[1, ::7] = -0.0                       # -0 ranks equal to +0
    q_pos = torch.full((T,), 4 * c, dtype=torch.int32, device="cuda")
    sel, n_sel, path = _gvr(q, scores, q_pos, K)
    assert host(path).tolist() == [3, 3]
    assert np.array_equal(host(sel), np.tile(np.arange(K, dtype=np.int32), (T, 1)))
    ref, _ = oracle.topk_groups(host(scores), host(q_pos), K)
    assert np.array_equal(host(sel), ref)


@pytest.mark.parametrize("K", [512, 2048])
def test_gvr_guess_missed_by_the_sample_is_caught(q, oracle, K):
    """Decode rows whose largest scores sit only at ids the strided sample
    never reads (i * c // 2048 is 31 mod 32 for c = 65,535): the guessed
    window lies far below the true K-th score, the exact counts reject it,
    and the row takes the cluster passes -- with the exact result."""
    T, c = 2, 65535
    g = torch.Generator(device="cpu").manual_seed(17)
    scores = torch.randn((T, c + 1), generator=g)
    hidden = torch.arange(7, c, 16)[: K + 100]
    scores[:, hidden] = 50.0 + torch.rand((T, hidden.numel()), generator=g)
    scores = scores.cuda()
    q_pos = torch.full((T,), 4 * c + 3, dtype=torch.int32, device="cuda")
    sel, n_sel, path = _gvr(q, scores, q_pos, K)
    assert host(path).tolist() == [3, 3]
    rs, rn = _radix(q, scores, q_pos, K)
    assert torch.equal(sel, rs) and torch.equal(n_sel, rn)
    ref, nref = oracle.topk_groups(host(scores), host(q_pos), K)
    assert np.array_equal(host(sel), ref) and np.array_equal(host(n_sel), nref)


@pytest.mark.parametrize("c, stride", [(131071, 131072), (100000, 100003), (250001, 262144)])
def test_gvr_cluster_rows_beyond_262k_tokens_and_odd_strides(q, oracle, c, stride):
    """Longer rows than the 262,144-token workload (32 and 64 keys per
    thread in the cluster) and a row stride that is not a multiple of 4
    (scalar loads): the self-sampled guess, against the radix Top-K and the
    oracle, at the three budgets."""
    T = 3
    g = torch.Generator(device="cpu").manual_seed(c % 1000)
    scores = torch.randn((T, stride), generator=g)
    scores[1] = torch.round(scores[1] * 4) / 4          # a row of many ties
    scores = scores.cuda()
    q_pos = torch.tensor([4 * c + 3, 4 * c, 4 * c + 1], dtype=torch.int32, device="cuda")
    for K in (512, 1024, 2048):
        sel, n_sel, path = _gvr(q, scores, q_pos, K)
        rs, rn = _radix(q, scores, q_pos, K)
        assert torch.equal(sel, rs) and torch.equal(n_sel, rn), K
        ref, nref = oracle.topk_groups(host(scores), host(q_pos), K)
        assert np.array_equal(host(sel), ref) and np.array_equal(host(n_sel), nref), K
        assert set(host(path).tolist()) <= {1, 3}


def test_gvr_other_budgets_use_the_radix_top_k(q):
    w = wl.b1_16k(device="cuda", K=300)
    st = QSAStep(w)
    st.index_scores()
    sel, n_sel, path = _gvr(q, st.scores, w.q_pos, 300)
    rs, rn = _radix(q, st.scores, w.q_pos, 300)
    assert torch.equal(sel, rs) and torch.equal(n_sel, rn)
    assert host(path).tolist() == [-1]          # untouched: the radix Top-K ran


def _rows_scores(T, stride, c, dist, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    s = torch.randn((T, stride), generator=g)
    if dist == "peaked":     # 5% of the groups 3 sigma up
        s += 3.0 * (torch.rand((T, stride), generator=g) < 0.05).float()
    elif dist == "ties":     # 16 levels
        s = torch.randint(0, 16, (T, stride), generator=g).float()
    q_pos = torch.full((T,), 4 * c + 2, dtype=torch.int32)
    return s.cuda(), q_pos.cuda()


@pytest.mark.parametrize("stride", [4096, 16384, 32768])     # 8, 32 and 64 keys per thread
@pytest.mark.parametrize("dist", ["normal", "peaked", "ties"])
def test_gvr_many_rows_one_cta_each(q, oracle, stride, dist):
    """Many rows (one CTA each, keys in registers): the self-sampled window
    selects on ordinary rows, bit for bit the radix Top-K and the oracle, at
    the three budgets; rows of the prefill chunk's length among them."""
    T, c = 160, stride - 1
    scores, q_pos = _rows_scores(T, stride, c, dist, seed=stride + len(dist))
    ref_s = host(scores)
    for K in (512, 1024, 2048):
        if K >= c:
            continue
        sel, n_sel, path = _gvr(q, scores, q_pos, K)
        rs, rn = _radix(q, scores, q_pos, K)
        assert torch.equal(sel, rs) and torch.equal(n_sel, rn), K
        ref, nref = oracle.topk_groups(ref_s, host(q_pos), K)
        assert np.array_equal(host(sel), ref) and np.array_equal(host(n_sel), nref), K
        p = host(path)
        if dist == "ties" or 4 * K > c:   # crowded levels; a K-th key near 0 (its window spans the sign)
            assert set(p.tolist()) <= {1, 3}, K
        else:
            assert np.all(p == 1), (K, np.bincount(p))


@pytest.mark.parametrize("K", [512, 2048])
def test_gvr_many_rows_guess_missed_by_the_sample_is_caught(q, oracle, K):
    """Rows of 16,383 candidates (32 keys per thread, every 8th id sampled)
    whose largest scores sit only at ids 3 mod 8: the window lies below
    them, the exact count above it exceeds the budget, and every row takes
    the radix passes -- with the exact result."""
    T, stride = 160, 16384
    c = stride - 1
    scores, q_pos = _rows_scores(T, stride, c, "normal", seed=K)
    hidden = torch.arange(3, c, 8)[: K + 100]
    scores[:, hidden.cuda()] = 50.0
    sel, n_sel, path = _gvr(q, scores, q_pos, K)
    assert np.all(host(path) == 3)
    rs, rn = _radix(q, scores, q_pos, K)
    assert torch.equal(sel, rs) and torch.equal(n_sel, rn)
    ref, nref = oracle.topk_groups(host(scores), host(q_pos), K)
    assert np.array_equal(host(sel), ref) and np.array_equal(host(n_sel), nref)
