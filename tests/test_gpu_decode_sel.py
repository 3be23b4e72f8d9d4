"""qsa_sparse_attn_decode_sel (stages 3 and 4 in one call) against the two
calls it replaces, qsa_expand_select then qsa_sparse_attn_decode, on the same
selection: out, lse and the status bits bit for bit.  The gather kernel's
own token listing (few rows), and the expand-into-workspace fallback of the
other plans (many rows on the streaming kernel; FP32 caches on the general
kernel); bad group ids and rows wider than W."""
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


def _two_calls(q, w, sel, n_sel, pos, W, cap):
    T = w.T
    tok = torch.empty((T, W), dtype=torch.int32, device="cuda")
    n_tok = torch.empty((T,), dtype=torch.int32, device="cuda")
    out = torch.empty((T, w.Hq, w.D), dtype=torch.float32 if w.q.dtype == torch.float32 else torch.bfloat16,
                      device="cuda")
    lse = torch.empty((T, w.Hq), dtype=torch.float32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    ws = torch.empty((max(q.qsa_sparse_attn_decode_workspace_size(T, w.Hq, w.Hkv, w.D, W, w.k_pages.dtype), 16),),
                     dtype=torch.uint8, device="cuda")
    q.qsa_expand_select(sel, n_sel, pos, tok, n_tok, capture_pos=cap, dev_status=status)
    q.qsa_sparse_attn_decode(w.q, w.k_pages, w.v_pages, w.page_table, tok, n_tok, out, workspace=ws,
                             k_scale=w.k_scale, v_scale=w.v_scale, q_req=w.q_req, lse=lse, dev_status=status)
    torch.cuda.synchronize()
    return out, lse, int(status.item())


def _fused(q, w, sel, n_sel, pos, W, cap):
    T = w.T
    out = torch.empty((T, w.Hq, w.D), dtype=torch.float32 if w.q.dtype == torch.float32 else torch.bfloat16,
                      device="cuda")
    lse = torch.empty((T, w.Hq), dtype=torch.float32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    need = q.qsa_sparse_attn_decode_sel_workspace_size(T, w.Hq, w.Hkv, w.D, W, w.k_pages.dtype)
    ws = torch.empty((max(need, 16),), dtype=torch.uint8, device="cuda")
    q.qsa_sparse_attn_decode_sel(w.q, w.k_pages, w.v_pages, w.page_table, sel, n_sel, pos, W, out, workspace=ws,
                                 capture_pos=cap, k_scale=w.k_scale, v_scale=w.v_scale, q_req=w.q_req, lse=lse,
                                 dev_status=status)
    torch.cuda.synchronize()
    return out, lse, int(status.item())


def _same(a, b):
    assert torch.equal(a[0], b[0]), float((a[0].float() - b[0].float()).abs().max())
    assert torch.equal(a[1], b[1])
    assert a[2] == b[2]


CASES = {   # name: workload; few rows take the gather kernel, the others a fallback
    "b8_fp8_gather": lambda: wl.make("sel_b8", B=8, ctx=65536, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512,
                                     kv_dtype="fp8", q_dtype="bf16", dist="peaked", seed=3, device="cuda"),
    "b2_bf16_gather_k2048": lambda: wl.make("sel_b2", B=2, ctx=16384, Hq=12, Hkv=1, D=256, H_I=4, D_I=128, K=2048,
                                            kv_dtype="bf16", q_dtype="bf16", dist="normal", seed=4, device="cuda"),
    "b80_fp8_streaming": lambda: wl.make("sel_b80", B=80, ctx=8192, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=128,
                                         kv_dtype="fp8", q_dtype="bf16", dist="peaked", seed=5, device="cuda"),
    "tiny_f32_general": lambda: wl.tiny(device="cuda"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fused_equals_expand_then_decode(q, name):
    w = CASES[name]()
    st = QSAStep(w)
    st.index_scores()
    st.topk()
    torch.cuda.synchronize()
    a = _two_calls(q, w, st.sel, st.n_sel, w.q_pos, w.W, None)
    b = _fused(q, w, st.sel, st.n_sel, w.q_pos, w.W, None)
    assert a[2] == 0
    _same(a, b)


def test_fused_with_capture_bad_groups_and_narrow_rows(q):
    """MTP reuse (capture 9 tokens back: two groups appended), a kept id at
    or above c(p0) (BAD_GROUP), and W cut one group short of a row (ROW_RANGE):
    the same outputs and status bits from both forms."""
    w = wl.make("sel_cap", B=4, ctx=16384, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512, kv_dtype="fp8",
                q_dtype="bf16", dist="peaked", seed=6, device="cuda")
    cap = (w.q_pos - 9).contiguous()
    st = QSAStep(w)
    st.sel_pos = cap
    st.index_scores()
    st.topk()
    torch.cuda.synchronize()
    sel = st.sel.clone()
    sel[1, 5] = int(host(cap)[1]) // 4 + 3          # not a candidate of the capture
    W_full = 4 * w.K + 4 + 4 * 3
    a = _two_calls(q, w, sel, st.n_sel, w.q_pos, W_full, cap)
    b = _fused(q, w, sel, st.n_sel, w.q_pos, W_full, cap)
    assert a[2] == q.QSA_DEV_BAD_GROUP
    _same(a, b)
    W_cut = 4 * w.K + 4                              # the appended groups no longer fit
    a = _two_calls(q, w, st.sel, st.n_sel, w.q_pos, W_cut, cap)
    b = _fused(q, w, st.sel, st.n_sel, w.q_pos, W_cut, cap)
    assert a[2] & q.QSA_DEV_ROW_RANGE
    _same(a, b)
