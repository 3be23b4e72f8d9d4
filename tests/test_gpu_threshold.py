"""The sequence-length threshold and its two decode graph families:
sequences of at most `threshold` tokens attend densely to every token (the
oracle's dense causal attention), longer ones through the QSA selection;
the dense and sparse CUDA graphs replay exactly what the eager calls do."""
import numpy as np
import pytest
import torch

from indexer_top_sparse_c4_b200 import workloads as wl
from indexer_top_sparse_c4_b200.pipeline import QSADecodeGraphs, QSAStep
from parity_utils import ATTN_MAX_ABS, ATTN_MEAN_ABS, ATTN_REL_L2, attn_errors, compact_pages, host, out_as_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from indexer_top_sparse_c4_b200 import build
    build.build()


def _mixed(K=512, thr=6000, kv="fp8"):
    # row 0: 1,500 tokens (dense by the budget itself), row 1: 5,000 (dense by
    # the threshold), rows 2, 3: 16,384 (QSA)
    pos = np.array([1499, 4999, 16383, 16383], np.int32)
    w = wl.make("thr", B=4, ctx=16384, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=K, kv_dtype=kv, q_dtype="bf16",
                dist="peaked", seed=13, device="cuda", q_pos=pos, q_req=np.arange(4, dtype=np.int32))
    return w, QSAStep(w, seq_len_threshold=thr)


def test_threshold_rows_are_dense_and_the_rest_sparse(oracle):
    w, st = _mixed()
    assert st.threshold == 6000 and st.w.W == 6000
    st.run()
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0
    tok, ntok = host(st.tok), host(st.n_tok)
    n = w.numpy()
    for t in (0, 1):
        p = int(n["q_pos"][t])
        assert ntok[t] == p + 1 and list(tok[t, :p + 1]) == list(range(p + 1))
    # the long rows: the oracle's QSA expansion of the GPU's selection
    sel_ref, nsel_ref = oracle.topk_groups(host(st.scores), n["q_pos"], w.K)
    tok_ref, ntok_ref, _ = oracle.expand_select(sel_ref, nsel_ref, n["q_pos"], st.w.W)
    for t in (2, 3):
        assert ntok[t] == ntok_ref[t] and np.array_equal(tok[t], tok_ref[t])
    kc, vc, pt = compact_pages(w.k_pages, w.v_pages, w.page_table, tok, ntok, n["q_req"])
    ref, _, sk = oracle.sparse_attn(n["q"], kc, vc, pt, tok, ntok, w.k_scale, w.v_scale, q_req=n["q_req"])
    assert sk == 0
    mx, mean, rel = attn_errors(out_as_f64(st.out), ref)
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel <= ATTN_REL_L2, (mx, mean, rel)


def test_graph_families_replay_the_eager_step():
    w, st = _mixed()
    g = QSADecodeGraphs(st)
    # a long batch: the sparse family
    st.run()
    torch.cuda.synchronize()
    eager = st.out.clone()
    st.out.zero_()
    assert g.replay(16384) == "sparse"
    torch.cuda.synchronize()
    assert torch.equal(st.out, eager)
    # a short batch (every sequence within the threshold): the dense family,
    # which launches no indexer or Top-K; same output as the eager dense calls
    w.q_pos.copy_(torch.tensor([1499, 4999, 5999, 777], dtype=torch.int32))
    st.dense_select(1 << 30)
    st.attention()
    torch.cuda.synchronize()
    eager = st.out.clone()
    st.out.zero_()
    st.tok.fill_(-7)
    assert g.replay(6000) == "dense"
    torch.cuda.synchronize()
    assert torch.equal(st.out, eager)
    assert int(st.status.item()) == 0
