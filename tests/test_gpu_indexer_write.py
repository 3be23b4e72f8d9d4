"""GPU parity of the steps before stage 1: the indexer projection (GEMV for
decode, tcgen05 GEMM for prefill) and the C4 compressed-key write, against
the oracle, through the C ABI; then the written keys feed stage 1 and 2."""
import numpy as np
import pytest
import torch

from indexer_top_sparse_c4_b200 import workloads as wl
from parity_utils import SCORE_REL, host, values_f64

pytestmark = pytest.mark.gpu

H_I, D_I = 4, 128
N = H_I * D_I + H_I + D_I      # 644 projected values per token


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from indexer_top_sparse_c4_b200 import build, qsa
    build.build()
    return qsa


def _projection_bound(x, w):
    """SCORE_REL * sum_h |x[t,h] w[n,h]|: the dot-product error scale."""
    return SCORE_REL * (np.abs(values_f64(x)) @ np.abs(values_f64(w)).T)


def _check_projection(q, oracle, T, H, x_dt="bf16", w_dt="bf16", rows=None, seed=0, n_rows=N):
    x = wl.hidden_states(T, H, seed=seed, device="cuda", dtype=x_dt)
    w, _, _ = wl.indexer_weights(H, H_I, D_I, seed=seed + 1, device="cuda", dtype=w_dt)
    w = w[:n_rows]
    y = torch.full((T, n_rows), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    q.qsa_indexer_project(x, w, y, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = list(range(T)) if rows is None else rows
    hx, hw = host(x)[rows], host(w)
    ref = oracle.indexer_project(hx, hw)
    got = host(y)[rows]
    assert np.isfinite(got).all()
    err = np.abs(got.astype(np.float64) - ref)
    assert np.all(err <= _projection_bound(hx, hw) + 1e-30), float(err.max())
    return x, w, y


@pytest.mark.parametrize("T", [1, 8, 13])
def test_projection_decode_gemv(q, oracle, T):
    """A handful of tokens (the decode step): the GEMV form, BF16 and FP32 mixes."""
    _check_projection(q, oracle, T, 5120)
    _check_projection(q, oracle, T, 1024, x_dt="f32", w_dt="bf16", seed=3)
    _check_projection(q, oracle, T, 512, x_dt="f32", w_dt="f32", seed=5)


@pytest.mark.parametrize("T", [3, 11])
def test_projection_gemv_hidden_chunks_and_ragged_rows(q, oracle, T):
    """Hidden sizes past one chunk of the GEMV's register-staged row (6,144
    columns for BF16 w, 4,096 for FP32 w), each with a ragged last chunk, and
    a row count that leaves the last CTA's four rows partly empty."""
    _check_projection(q, oracle, T, 8200, seed=11)
    _check_projection(q, oracle, T, 4104, x_dt="f32", w_dt="f32", seed=13)
    _check_projection(q, oracle, T, 2048, seed=15, n_rows=641)


def test_projection_prefill_tensor_cores_ragged(q, oracle):
    """The tcgen05 GEMM on a token count and a row count that are not
    multiples of its 128 x 128 tiles: every row checked."""
    _check_projection(q, oracle, 1000, 1024)


def test_projection_prefill_chunk_sampled(q, oracle):
    """8,192 tokens x 5,120 hidden (the prefill chunk's size): one row of
    every 128-token tile, at a different offset in each."""
    rows = [128 * i + (41 * i) % 128 for i in range(64)]
    _check_projection(q, oracle, 8192, 5120, rows=rows)


def _pages_with_sentinel(num_pages, dt, d=D_I):
    if dt == "f32":
        return torch.full((num_pages, 16, d), 7.0, dtype=torch.float32, device="cuda")
    return torch.full((num_pages, 16, d), 7.0, dtype=torch.bfloat16, device="cuda")


def _check_compress(q, oracle, k_tok, g_id, g_req, pt, num_pages, dt, seed=0, weights=None):
    d = k_tok.shape[1]
    _, wphi, bias = wl.indexer_weights(256, H_I, d, seed=seed, device="cuda") if weights is None else weights
    pages = _pages_with_sentinel(num_pages, dt, d)
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    q.qsa_compress_keys(k_tok, g_id, wphi, pages, pt, g_req=g_req, bias=bias, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    want = host(_pages_with_sentinel(num_pages, dt, d))
    kt = host(k_tok.contiguous()).reshape(-1, 4, d)
    skipped = oracle.compress_keys(kt, host(g_id), host(wphi), want, host(pt),
                                   g_req=None if g_req is None else host(g_req), bias=host(bias))
    assert skipped == 0
    got = host(pages)
    # rows no group maps to are untouched, bit for bit
    written = np.zeros((num_pages, 16), bool)
    pt_h, gid_h = host(pt), host(g_id)
    req_h = np.zeros_like(gid_h) if g_req is None else host(g_req)
    for r, g in zip(req_h, gid_h):
        written[pt_h[r, g // 16], g % 16] = True
    assert np.array_equal(got[~written], want[~written])
    # written rows: within the dot-product bound; with BF16 storage both sides
    # round values that differ within that bound, so they may land on
    # neighbouring BF16 values: one step, at most |v| * 2^-7
    wphi_h, b_h = host(wphi).astype(np.float64), host(bias).astype(np.float64)
    for i, (r, g) in enumerate(zip(req_h, gid_h)):
        p, row = pt_h[r, g // 16], g % 16
        scale = np.abs(wphi_h) @ np.abs(kt[i].reshape(-1).astype(np.float64)) + np.abs(b_h)
        gv, wv = values_f64(got[p, row]), values_f64(want[p, row])
        tol = SCORE_REL * scale + (np.abs(wv) * 2.0 ** -7 if dt == "bf16" else 0.0)
        assert np.all(np.abs(gv - wv) <= tol + 1e-30), (i, float(np.abs(gv - wv).max()))
    return pages


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_compress_prefill_chunk_in_place(q, oracle, dt):
    """A 2,048-token chunk starting at a group boundary: its 512 groups read
    straight from the projection output (the token-key columns, row stride
    N), written through a permuted page table."""
    T, H = 2048, 1024
    x = wl.hidden_states(T, H, seed=7, device="cuda")
    w, _, _ = wl.indexer_weights(H, H_I, D_I, seed=8, device="cuda")
    y = torch.empty((T, N), dtype=torch.float32, device="cuda")
    q.qsa_indexer_project(x, w, y)
    k_tok = y[:, H_I * D_I + H_I:]                      # [T, D_I], row stride N
    pages_per_req = 64
    g = torch.Generator(device="cpu").manual_seed(9)
    pt = torch.randperm(pages_per_req, generator=g).to(torch.int32).view(1, -1).cuda()
    # the chunk follows a 1,024-token prefix: its groups are 256 .. 767 (logical pages 16 .. 47)
    g_id = torch.arange(256, 256 + T // 4, dtype=torch.int32, device="cuda")
    _check_compress(q, oracle, k_tok, g_id, None, pt, pages_per_req, dt)


@pytest.mark.parametrize("d", [32, 64, 128])
def test_compress_dims_unaligned_operands_ragged_groups(q, oracle, d):
    """Every built D_I, 37 groups (two full CTAs of 16 and a ragged third),
    token-key rows at an odd stride and a W_phi that does not start on a
    16-byte boundary: the 4-byte copy paths."""
    n = 37
    gen = torch.Generator(device="cpu").manual_seed(40 + d)
    buf = torch.randn((4 * n, d + 3), generator=gen).cuda()
    k_tok = buf[:, :d]                                     # row stride d + 3
    _, wphi, bias = wl.indexer_weights(256, H_I, d, seed=41, device="cuda")
    raw = torch.empty((wphi.numel() + 1,), dtype=torch.float32, device="cuda")
    wphi_odd = raw[1:].view(wphi.shape)
    wphi_odd.copy_(wphi)
    assert wphi_odd.data_ptr() % 16 != 0 and k_tok.stride(0) % 4 != 0
    P = 8
    pt = torch.randperm(P, generator=gen).to(torch.int32).view(1, -1).cuda()
    g_id = torch.randperm(P * 16, generator=gen)[:n].to(torch.int32).cuda()
    _check_compress(q, oracle, k_tok, g_id, None, pt, P, "f32", weights=(None, wphi_odd, bias))
    _check_compress(q, oracle, k_tok, g_id, None, pt, P, "bf16", weights=(None, wphi_odd, bias))


def test_compress_decode_ring(q, oracle):
    """Decode: each of 8 requests completed one group this step; its four
    token keys come from a per-request ring [B, 4, D_I]."""
    B = 8
    ring = torch.randn((B * 4, D_I), generator=torch.Generator(device="cpu").manual_seed(11)).cuda()
    g_id = torch.tensor([65534, 3, 17, 4095, 100, 0, 16, 31], dtype=torch.int32, device="cuda")
    g_req = torch.arange(B, dtype=torch.int32, device="cuda")
    P = 4096
    pt = torch.randperm(B * P, generator=torch.Generator(device="cpu").manual_seed(12)).to(torch.int32)
    pt = pt.view(B, P).cuda()
    _check_compress(q, oracle, ring, g_id, g_req, pt, B * P, "f32")


def test_compress_flags_and_skips_bad_ids(q):
    """A request outside the page table, a negative group and a bad physical
    page raise their status bits; those groups are not written."""
    k_tok = torch.ones((4 * 4, D_I), dtype=torch.float32, device="cuda")
    _, wphi, bias = wl.indexer_weights(64, H_I, D_I, seed=1, device="cuda")
    pt = torch.tensor([[0, 1], [2, 77]], dtype=torch.int32, device="cuda")
    g_req = torch.tensor([0, 5, 0, 1], dtype=torch.int32, device="cuda")
    g_id = torch.tensor([3, 3, -1, 20], dtype=torch.int32, device="cuda")   # only the first is good
    pages = _pages_with_sentinel(3, "f32")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    q.qsa_compress_keys(k_tok, g_id, wphi, pages, pt, g_req=g_req, bias=bias, dev_status=status)
    torch.cuda.synchronize()
    st = int(status.item())
    assert st & q.QSA_DEV_BAD_REQUEST and st & q.QSA_DEV_BAD_GROUP and st & q.QSA_DEV_BAD_PAGE
    changed = (pages != 7.0).any(dim=-1)
    assert changed.sum().item() == 1 and bool(changed[0, 3])


def test_written_keys_feed_the_indexer(q, oracle):
    """Hidden states -> projection -> compressed keys written into pages ->
    stage 1 scores (query and head weights from the same projection) ->
    stage 2: scores within the dot-product bound of the oracle's scores on
    the written keys, Top-K bit-exact on the GPU's scores."""
    from parity_utils import score_bound
    T_ctx, H, B = 4096, 1024, 1
    groups = T_ctx // 4
    x = wl.hidden_states(T_ctx, H, seed=21, device="cuda")
    w, wphi, bias = wl.indexer_weights(H, H_I, D_I, seed=22, device="cuda")
    y = torch.empty((T_ctx, N), dtype=torch.float32, device="cuda")
    q.qsa_indexer_project(x, w, y)
    P = T_ctx // 64
    pt = torch.randperm(P, generator=torch.Generator(device="cpu").manual_seed(23)).to(torch.int32)
    pt = pt.view(1, P).cuda()
    pages = torch.zeros((P, 16, D_I), dtype=torch.float32, device="cuda")
    g_id = torch.arange(groups, dtype=torch.int32, device="cuda")
    q.qsa_compress_keys(y[:, H_I * D_I + H_I:], g_id, wphi, pages, pt, bias=bias)
    # the last token queries every complete group before its own block
    t = T_ctx - 1
    q_idx = y[t:t + 1, :H_I * D_I].reshape(1, H_I, D_I).contiguous()
    w_idx = y[t:t + 1, H_I * D_I:H_I * D_I + H_I].contiguous()
    q_pos = torch.tensor([t], dtype=torch.int32, device="cuda")
    q_req = torch.zeros((1,), dtype=torch.int32, device="cuda")
    stride = groups
    scores = torch.empty((1, stride), dtype=torch.float32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    q.qsa_index_scores(q_idx, w_idx, pages, pt, q_pos, scores, q_req=q_req, dev_status=status)
    K = 64
    sel = torch.empty((1, K), dtype=torch.int32, device="cuda")
    n_sel = torch.empty((1,), dtype=torch.int32, device="cuda")
    q.qsa_topk_groups(scores, q_pos, K, sel, n_sel, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    n = {k: host(v) for k, v in dict(q_idx=q_idx, w_idx=w_idx, pages=pages, pt=pt, q_pos=q_pos,
                                     q_req=q_req).items()}
    ref, skipped = oracle.index_scores(n["q_idx"], n["w_idx"], n["pages"], n["pt"], n["q_pos"], n["q_req"], stride)
    assert skipped == 0
    c = t // 4
    bound = score_bound(n["q_idx"], n["w_idx"], n["pages"], n["pt"], n["q_req"], n["q_pos"], [0], stride)
    gs = host(scores)
    assert np.all(np.abs(gs[0, :c].astype(np.float64) - ref[0, :c]) <= bound[0, :c] + 1e-30)
    sel_ref, nsel_ref = oracle.topk_groups(gs, n["q_pos"], K)
    assert np.array_equal(host(sel), sel_ref) and np.array_equal(host(n_sel), nsel_ref)
