"""qsa_sparse_attn_decode_noalloc: the decode attention for callers that cannot
allocate device memory (a graph capture that must not allocate, a fully
carved-up memory pool, a plugin handed only its inputs and outputs).  It must
give the same results as qsa_sparse_attn_decode with a caller workspace, call
after call, although every call reuses the library's one scratch buffer.

Kept in a file of its own that pytest collects last."""
import numpy as np
import pytest
import torch

from parity_utils import ATTN_MAX_ABS, ATTN_MEAN_ABS, ATTN_REL_L2, attn_errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from indexer_top_sparse_c4_b200 import build, qsa
    build.build()
    return qsa


def _selection(w):
    from indexer_top_sparse_c4_b200.pipeline import QSAStep
    step = QSAStep(w)
    step.run()                       # decode through the workspace entry point
    torch.cuda.synchronize()
    return step


@pytest.mark.parametrize("which", ["b1_16k_bf16_k2048", "b2_16k_fp8_k4096"])
def test_noalloc_matches_workspace_decode_on_two_calls(lib, which):
    # rows too long for one cluster (8,196 BF16 / 16,388 FP8 token slots) are
    # split over CTA groups whose partials go through the scratch buffer
    from indexer_top_sparse_c4_b200 import workloads as wl
    make = (lambda s: wl.b1_16k(device="cuda", seed=s, K=2048)) if which == "b1_16k_bf16_k2048" else \
        (lambda s: wl.b1_16k(device="cuda", seed=s, B=2, kv_dtype="fp8", K=4096))
    for seed in (11, 12):            # two calls in a row, different inputs each time
        w = make(seed)
        step = _selection(w)
        need = lib.qsa_sparse_attn_decode_workspace_size(w.T, w.Hq, w.Hkv, w.D, w.W, w.k_pages.dtype)
        assert 0 < need <= 32 * 1024 * 1024  # per-CTA partials: scratch in use
        out = torch.full_like(step.out, float("nan"))
        lse = torch.full_like(step.lse, float("nan"))
        status = torch.zeros((1,), dtype=torch.int32, device="cuda")
        lib.qsa_sparse_attn_decode_noalloc(w.q, w.k_pages, w.v_pages, w.page_table, step.tok,
                                           step.n_tok, out, k_scale=w.k_scale, v_scale=w.v_scale,
                                           q_req=w.q_req, lse=lse, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref = step.out.double().cpu().numpy()
        got = out.double().cpu().numpy()
        mx, mean, rel = attn_errors(got, ref)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel <= ATTN_REL_L2, (mx, mean, rel)
        assert torch.allclose(lse, step.lse, atol=1e-3, rtol=0)


def test_noalloc_refuses_shapes_beyond_its_buffer(lib):
    # 64 queries x 16 heads x 129 chunk partials of 256 floats exceed 32 MiB
    T, Hq, Hkv, D, W = 64, 16, 2, 256, 8196
    assert lib.qsa_sparse_attn_decode_workspace_size(T, Hq, Hkv, D, W, torch.uint8) > 32 * 1024 * 1024
    q = torch.zeros((T, Hq, D), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1, 64, Hkv, D), dtype=torch.uint8, device="cuda")  # FP8 codes
    pt = torch.zeros((T, 1), dtype=torch.int32, device="cuda")
    tok = torch.full((T, W), -1, dtype=torch.int32, device="cuda")
    n_tok = torch.zeros((T,), dtype=torch.int32, device="cuda")
    out = torch.empty((T, Hq, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.QSAError, match="built-in buffer"):
        lib.qsa_sparse_attn_decode_noalloc(q, kv, kv, pt, tok, n_tok, out, k_scale=1.0, v_scale=1.0)
