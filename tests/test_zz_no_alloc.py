"""qsa_sparse_attn_decode_noalloc: the decode attention for callers that cannot
allocate device memory (a graph capture that must not allocate, a fully
carved-up memory pool, a plugin handed only its inputs and outputs).  It runs
the same plan and kernels as qsa_sparse_attn_decode with a caller workspace,
so its outputs must be bit-identical to that call's, call after call, although
every call reuses the library's one scratch buffer.

Kept in a file of its own that pytest collects last."""
import pytest
import torch

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


def _noalloc(lib, w, step):
    out = torch.full_like(step.out, float("nan"))
    lse = torch.full_like(step.lse, float("nan"))
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    lib.qsa_sparse_attn_decode_noalloc(w.q, w.k_pages, w.v_pages, w.page_table, step.tok,
                                       step.n_tok, out, k_scale=w.k_scale, v_scale=w.v_scale,
                                       q_req=w.q_req, lse=lse, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, lse


def test_noalloc_matches_workspace_decode_on_two_calls(lib):
    """Two calls in a row: the first with rows long enough to need many
    partials in the scratch, the second with fewer.  A read of the first
    call's leftover partials by the second would change its output."""
    from indexer_top_sparse_c4_b200 import workloads as wl
    shapes = [
        lambda: wl.b1_16k(device="cuda", seed=11, B=2, kv_dtype="fp8", K=4096),   # 4 rows of 16,388 slots
        lambda: wl.b1_16k(device="cuda", seed=12, K=512),                          # 2 rows of 2,052 slots
    ]
    needs = []
    for make in shapes:
        w = make()
        step = _selection(w)
        need = lib.qsa_sparse_attn_decode_workspace_size(w.T, w.Hq, w.Hkv, w.D, w.W, w.k_pages.dtype)
        assert 0 < need <= 32 * 1024 * 1024   # the scratch is in use
        needs.append(need)
        out, lse = _noalloc(lib, w, step)
        assert torch.equal(out, step.out)
        assert torch.equal(lse, step.lse)
    assert needs[1] < needs[0]


def test_noalloc_refuses_shapes_beyond_its_buffer(lib):
    # 2 queries x 16 heads x 1,024 chunk partials (rows of 2^20 slots, 1,024
    # slots per chunk) of 258 floats exceed 32 MiB
    T, Hq, Hkv, D, W = 2, 16, 1, 256, 1 << 20
    assert lib.qsa_sparse_attn_decode_workspace_size(T, Hq, Hkv, D, W, torch.uint8) > 32 * 1024 * 1024
    q = torch.zeros((T, Hq, D), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1, 64, Hkv, D), dtype=torch.uint8, device="cuda")  # FP8 codes
    pt = torch.zeros((T, 1), dtype=torch.int32, device="cuda")
    tok = torch.full((T, W), -1, dtype=torch.int32, device="cuda")
    n_tok = torch.zeros((T,), dtype=torch.int32, device="cuda")
    out = torch.empty((T, Hq, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.QSAError, match="built-in buffer"):
        lib.qsa_sparse_attn_decode_noalloc(q, kv, kv, pt, tok, n_tok, out, k_scale=1.0, v_scale=1.0)


def test_noalloc_reports_bad_arguments_before_the_scratch_size(lib):
    """A shape that is invalid (Hq not a multiple of Hkv) and would also need
    more scratch than the buffer holds is refused as an invalid argument."""
    T, Hq, Hkv, D, W = 2, 15, 2, 256, 1 << 20
    q = torch.zeros((T, Hq, D), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1, 64, Hkv, D), dtype=torch.uint8, device="cuda")
    pt = torch.zeros((T, 1), dtype=torch.int32, device="cuda")
    tok = torch.full((T, W), -1, dtype=torch.int32, device="cuda")
    n_tok = torch.zeros((T,), dtype=torch.int32, device="cuda")
    out = torch.empty((T, Hq, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.QSAError) as e:
        lib.qsa_sparse_attn_decode_noalloc(q, kv, kv, pt, tok, n_tok, out, k_scale=1.0, v_scale=1.0)
    assert e.value.status == lib.QSA_ERR_INVALID_ARG
