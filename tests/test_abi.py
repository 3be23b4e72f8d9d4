"""The C-ABI library: it builds for sm_100a, loads, exports every entry point
the header declares, and rejects bad arguments on the host before any launch.
No GPU needed: every call here fails validation (or has T == 0) before it
touches the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from indexer_top_sparse_c4_b200 import build, qsa
    build.build()
    return qsa.lib()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^QSA_API\s+[\w\s\*]+?\b(qsa_\w+)\s*\(", src, re.M))
    return sorted(names)


def test_header_declares_the_five_calls():
    names = declared_symbols()
    for n in ("qsa_index_scores", "qsa_topk_groups", "qsa_expand_select",
              "qsa_sparse_attn_decode", "qsa_sparse_attn_prefill"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    from indexer_top_sparse_c4_b200 import qsa
    for n in declared_symbols():
        assert hasattr(L, n), n
    assert set(qsa.ENTRY_POINTS) <= set(declared_symbols())
    assert L.qsa_abi_version() == 11


def test_library_has_no_torch_or_python_dependency():
    from indexer_top_sparse_c4_b200 import build
    import subprocess
    out = subprocess.run(["ldd", build.LIB], capture_output=True, text=True).stdout
    assert "torch" not in out and "python" not in out and "cudart" not in out


def _err(L):
    return L.qsa_last_error_string().decode()


NULL = None


def test_index_scores_rejects_unbuilt_shapes(L):
    st = L.qsa_index_scores(NULL, 0, NULL, NULL, 0, 1, NULL, 1, 1, NULL, NULL, 4, 3, 128, NULL, 16, NULL, NULL, NULL)
    assert st == 2 and "H_I" in _err(L)
    st = L.qsa_index_scores(NULL, 0, NULL, NULL, 0, 1, NULL, 1, 1, NULL, NULL, -1, 4, 128, NULL, 16, NULL, NULL, NULL)
    assert st == 1
    st = L.qsa_index_scores(NULL, 0, NULL, NULL, 0, 1, NULL, 1, 1, NULL, NULL, 4, 4, 128, NULL, 16, NULL, NULL, NULL)
    assert st == 1 and "null" in _err(L)
    st = L.qsa_index_scores(NULL, 2, NULL, NULL, 0, 1, NULL, 1, 1, NULL, NULL, 4, 4, 128, NULL, 16, NULL, NULL, NULL)
    assert st == 1 and "dtype" in _err(L)
    # T == 0 is a no-op that launches nothing
    assert L.qsa_index_scores(NULL, 0, NULL, NULL, 0, 1, NULL, 1, 1, NULL, NULL, 0, 4, 128, NULL, 16, NULL, NULL, NULL) == 0


def test_index_scores_rejects_misaligned_pointers(L):
    bad = ctypes.c_void_p(0x1004)
    ok = ctypes.c_void_p(0x2000)
    st = L.qsa_index_scores(bad, 0, ok, ok, 0, 1, ok, 1, 1, NULL, ok, 1, 4, 128, ok, 16, NULL, NULL, NULL)
    assert st == 1 and "aligned" in _err(L)


def test_prefix_hist_must_be_aligned(L):
    ok = ctypes.c_void_p(0x2000)
    bad = ctypes.c_void_p(0x2008)
    st = L.qsa_index_scores(ok, 0, ok, ok, 0, 1, ok, 1, 1, NULL, ok, 1, 4, 128, ok, 16, bad, NULL, NULL)
    assert st == 1 and "prefix_hist" in _err(L)
    assert L.qsa_topk_groups(ok, 16, bad, ok, 1, 4, ok, ok, NULL, 0, NULL, NULL) == 1
    assert "prefix_hist" in _err(L)
    assert L.qsa_topk_expand(ok, 16, bad, ok, 1, 4, ok, ok, ok, ok, 20, NULL, NULL) == 1
    assert "prefix_hist" in _err(L)


def test_topk_validation(L):
    assert L.qsa_topk_groups(NULL, 16, NULL, NULL, 2, 0, NULL, NULL, NULL, 0, NULL, NULL) == 1
    assert L.qsa_topk_groups(NULL, 0, NULL, NULL, 2, 4, NULL, NULL, NULL, 0, NULL, NULL) == 1
    assert L.qsa_topk_groups(NULL, 10 ** 7, NULL, NULL, 2, 4, NULL, NULL, NULL, 0, NULL, NULL) == 2
    assert L.qsa_topk_groups(NULL, 16, NULL, NULL, 0, 4, NULL, NULL, NULL, 0, NULL, NULL) == 0
    assert L.qsa_topk_groups_workspace_size(8, 512, 65535) == 0
    # rows of up to 262,144 candidates (8 CTAs x 512 threads x 64 keys)
    assert L.qsa_topk_groups(NULL, 262144, NULL, NULL, 0, 4, NULL, NULL, NULL, 0, NULL, NULL) == 0
    assert L.qsa_topk_groups(NULL, 262145, NULL, NULL, 0, 4, NULL, NULL, NULL, 0, NULL, NULL) == 2
    assert L.qsa_topk_groups_gvr(NULL, 262144, NULL, 0, 512, NULL, NULL, NULL, NULL, NULL) == 0
    assert L.qsa_topk_groups_gvr(NULL, 262145, NULL, 0, 512, NULL, NULL, NULL, NULL, NULL) == 2
    assert L.qsa_topk_groups_gvr(NULL, 16, NULL, 2, 512, NULL, NULL, NULL, NULL, NULL) == 1   # null pointers


def test_expand_validation(L):
    assert L.qsa_expand_select(NULL, NULL, 8, NULL, NULL, 1, NULL, NULL, 35, NULL, NULL) == 1
    assert "4*K + 4" in _err(L)
    assert L.qsa_expand_select(NULL, NULL, 8, NULL, NULL, 1, NULL, NULL, 36, NULL, NULL) == 1
    assert L.qsa_expand_select(NULL, NULL, 8, NULL, NULL, 0, NULL, NULL, 36, NULL, NULL) == 0


def test_topk_expand_validation(L):
    # (scores, stride, prefix_hist, q_pos, T, K, sel, n_sel, tok, n_tok, W, status, stream)
    assert L.qsa_topk_expand(NULL, 16, NULL, NULL, 1, 8, NULL, NULL, NULL, NULL, 35, NULL, NULL) == 1
    assert "4*K + 4" in _err(L)
    assert L.qsa_topk_expand(NULL, 16, NULL, NULL, 1, 0, NULL, NULL, NULL, NULL, 36, NULL, NULL) == 1
    assert L.qsa_topk_expand(NULL, 10 ** 7, NULL, NULL, 1, 8, NULL, NULL, NULL, NULL, 36, NULL, NULL) == 2
    assert L.qsa_topk_expand(NULL, 16, NULL, NULL, 1, 8, NULL, NULL, NULL, NULL, 36, NULL, NULL) == 1
    assert "null" in _err(L)
    assert L.qsa_topk_expand(NULL, 16, NULL, NULL, 0, 8, NULL, NULL, NULL, NULL, 36, NULL, NULL) == 0


def _attn(L, fn, T=1, Hq=16, Hkv=2, D=256, kv_dt=1, q_dt=1, out_dt=1, W=36, ks=1.0, vs=1.0,
          ptr=NULL, ws=NULL, ws_bytes=0):
    args = [ptr, q_dt, ptr, ptr, kv_dt, ks, vs, 4, ptr, 1, 1, NULL, ptr, ptr, W, T, Hq, Hkv, D, 0.0, ptr,
            out_dt, NULL]
    if fn == "decode":
        return L.qsa_sparse_attn_decode(*args, ws, ws_bytes, NULL, NULL)
    return L.qsa_sparse_attn_prefill(*args, NULL, NULL)


@pytest.mark.parametrize("fn", ["decode", "prefill"])
def test_attention_validation(L, fn):
    assert _attn(L, fn, D=96) == 2 and "head dim" in _err(L)
    assert _attn(L, fn, Hq=17, Hkv=1) == 2
    assert _attn(L, fn, Hq=6, Hkv=4) == 1
    assert _attn(L, fn, kv_dt=2, ks=0.0) == 1 and "FP8" in _err(L)
    assert _attn(L, fn, q_dt=2) == 1
    assert _attn(L, fn) == 1 and "null" in _err(L)
    assert _attn(L, fn, T=0) == 0
    assert _attn(L, fn, T=70000) == 2


def test_decode_workspace_is_checked(L):
    # many (query, KV head) rows (prefill-sized T) need no workspace; a decode
    # batch spreads each row over several CTAs whose partials go through it
    assert L.qsa_sparse_attn_decode_workspace_size(8192, 24, 2, 256, 2052, 1) == 0
    need = L.qsa_sparse_attn_decode_workspace_size(8, 16, 2, 256, 2052, 2)
    assert need > 0 and need == 8 * 16 * 9 * (256 + 2) * 4   # 9 chunks per row: 144 CTAs
    need = L.qsa_sparse_attn_decode_workspace_size(1, 16, 2, 256, 8196, 1)
    assert need > 0
    ok = ctypes.c_void_p(0x10000)
    st = _attn(L, "decode", T=1, W=8196, ptr=ok, ws=ok, ws_bytes=need - 16)
    assert st == 3 and str(need) in _err(L)


def test_decode_sel_validation(L):
    """The fused stage 3 + 4 call: W below 4K + 4 and a missing or short
    workspace are refused on the host, before any launch."""
    P, I, F, U = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    f = L.qsa_sparse_attn_decode_sel
    f.argtypes = [P, I, P, P, I, F, F, I, P, I, I, P, P, P, I, P, P, I, I, I, I, I, F, P, I, P, P, U, P, P]
    L.qsa_sparse_attn_decode_sel_workspace_size.restype = U
    L.qsa_sparse_attn_decode_sel_workspace_size.argtypes = [I, I, I, I, I, I]
    ok = ctypes.c_void_p(0x10000)

    def call(K=512, W=2052, T=8, ws=ok, ws_bytes=1 << 30):
        # (q, q_dt, k, v, kv_dt, ks, vs, pages, pt, pt_rows, pt_stride, q_req, sel, n_sel, K, q_pos, cap,
        #  W, T, Hq, Hkv, D, sm_scale, out, out_dt, lse, ws, ws_bytes, status, stream)
        return f(ok, 1, ok, ok, 2, 1.0, 1.0, 4096, ok, 8, 4096, NULL, ok, ok, K, ok, NULL, W, T, 16, 2, 256, 0.0,
                 ok, 1, NULL, ws, ws_bytes, NULL, NULL)
    assert call(W=2051) == 1 and "W must be" in _err(L)
    assert call(K=0) == 1
    need = L.qsa_sparse_attn_decode_sel_workspace_size(8, 16, 2, 256, 2052, 2)
    assert need == L.qsa_sparse_attn_decode_workspace_size(8, 16, 2, 256, 2052, 2)   # the gather plan
    assert call(ws_bytes=need - 16) == 3 and str(need) in _err(L)
    assert call(ws=NULL) == 3
    # many rows: the token lists go through the workspace too
    big = L.qsa_sparse_attn_decode_sel_workspace_size(200, 16, 2, 256, 2052, 2)
    assert big >= 200 * 2052 * 4


def test_bind_records_launches_and_checks_them_when_called(L):
    """qsa.bind: the wrapped wrapper runs once with the library's launching
    calls recorded, not made; the bound call makes them, and a call the
    library refuses raises then, not at binding.  Size queries are answered
    at binding and not recorded."""
    import torch
    from indexer_top_sparse_c4_b200 import qsa

    class Stream:
        cuda_stream = 0

    scores = torch.zeros((1, 8))
    q_pos = torch.zeros((1,), dtype=torch.int32)
    sel = torch.zeros((1, 1), dtype=torch.int32)
    n_sel = torch.zeros((1,), dtype=torch.int32)
    call = qsa.bind(qsa.qsa_topk_groups_gvr, scores, q_pos, 0, sel, n_sel, stream=Stream())   # K = 0
    with pytest.raises(qsa.QSAError, match="K must be"):
        call()
    empty = torch.zeros((0, 4), dtype=torch.int32)
    qsa.bind(qsa.qsa_dense_select, torch.zeros((0,), dtype=torch.int32), 100, empty,
             torch.zeros((0,), dtype=torch.int32), stream=Stream())()          # T = 0: nothing to launch
    sizes = []
    nothing = qsa.bind(lambda: sizes.append(qsa.qsa_sparse_attn_decode_workspace_size(8, 16, 2, 256, 2052, 2)))
    assert sizes == [L.qsa_sparse_attn_decode_workspace_size(8, 16, 2, 256, 2052, 2)] and sizes[0] > 0
    nothing()
    assert qsa.lib() is L                                # binding leaves the library in place


@pytest.mark.parametrize("T, Hq, Hkv, D, W, kv, parts", [
    (8, 16, 2, 256, 2052, 2, 9),      # B8, K=512: 16 rows, one CTA per SM -> 9 chunks per row
    (8, 16, 2, 256, 8196, 2, 9),      # K=2,048: the same 9 chunks, longer
    (8, 16, 2, 256, 16388, 2, 17),    # K=4,096: the row-index table (1,024 slots) forces 17 chunks
    (40, 16, 2, 256, 2052, 2, 3),     # 80 rows: one per SM would do, the table asks for 3
    (40, 16, 2, 256, 516, 2, 1),      # 80 rows of 516 slots: one chunk each, no partials
    (80, 16, 2, 256, 2052, 2, 1),     # 160 rows: the streaming kernel, no partials
    (1, 4, 1, 64, 132, 0, 3),         # FP32 / D=64: the general kernel, split in 64-slot pieces
])
def test_decode_plan_through_the_workspace_query(L, T, Hq, Hkv, D, W, kv, parts):
    """The decode attention's plan, seen through its workspace: T * Hq
    partials of (D + 2) floats per chunk (or split) of a row, none when a
    row is not split."""
    need = L.qsa_sparse_attn_decode_workspace_size(T, Hq, Hkv, D, W, kv)
    assert need == (0 if parts == 1 else T * Hq * parts * (D + 2) * 4)
    sel = L.qsa_sparse_attn_decode_sel_workspace_size(T, Hq, Hkv, D, W, kv)
    gather = kv != 0 and T * Hkv < 148
    if gather:   # the gather kernel lists its tokens itself
        assert sel == need
    else:        # the token lists go through the workspace
        a16 = lambda n: (n + 15) // 16 * 16
        assert sel == a16(need) + a16(T * W * 4) + a16(T * 4)


def test_binding_refuses_to_run_without_the_library(monkeypatch, tmp_path):
    from indexer_top_sparse_c4_b200 import qsa
    monkeypatch.setattr(qsa, "LIB_PATH", str(tmp_path / "libqsa.so"))
    monkeypatch.setattr(qsa, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        qsa.lib()


def test_every_stage_has_a_workspace_query(L):
    """The stages that keep their state on chip report 0 bytes."""
    from indexer_top_sparse_c4_b200 import qsa
    assert L.qsa_index_scores_workspace_size(8, 4, 128, 65535) == 0
    assert L.qsa_index_scores_workspace_size(8192, 4, 128, 16384) == 0
    assert L.qsa_expand_select_workspace_size(8, 512, 2052) == 0
    assert L.qsa_sparse_attn_prefill_workspace_size(8192, 24, 2, 256, 2052, 1) == 0
    for name in ("index_scores", "topk_groups", "expand_select", "sparse_attn_decode",
                 "sparse_attn_prefill"):
        assert f"qsa_{name}_workspace_size" in qsa.ENTRY_POINTS


def test_status_codes_have_names(L):
    names = {i: L.qsa_status_name(i).decode() for i in range(7)}
    assert names[5] == "QSA_ERR_DEVICE_INDEX" and names[6] == "QSA_ERR_TIMEOUT"
    assert L.qsa_status_name(99).decode() == "QSA_ERR_UNKNOWN"


def test_device_status_query_checks_its_pointer(L):
    """A null or misaligned status word is refused on the host (no copy)."""
    bits = ctypes.c_uint32(7)
    assert L.qsa_get_device_status(NULL, ctypes.byref(bits), 0, NULL) == 1
    assert "NULL" in _err(L)
    assert L.qsa_get_device_status(ctypes.c_void_p(0x2002), ctypes.byref(bits), 1, NULL) == 1
    assert "aligned" in _err(L)
    assert bits.value == 7


def test_bounded_wait_selftest_validation(L):
    """The self-test refuses null pointers and limits outside 1 us .. 1 s on
    the host, before any launch."""
    ok = ctypes.c_void_p(0x2000)
    f = L.qsa_selftest_bounded_wait
    f.argtypes = [ctypes.c_uint32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    assert f(1000, NULL, ok, NULL) == 1 and "null" in _err(L)
    assert f(1000, ok, NULL, NULL) == 1
    assert f(0, ok, ok, NULL) == 1 and "limit_us" in _err(L)
    assert f(1000001, ok, ok, NULL) == 1 and "limit_us" in _err(L)


def test_indexer_write_validation(L):
    ok = ctypes.c_void_p(0x2000)
    # (x, x_dt, w, w_dt, T, H, N, y, status, stream)
    assert L.qsa_indexer_project(ok, 1, ok, 1, 8, 5120, 0, ok, NULL, NULL) == 1
    assert L.qsa_indexer_project(ok, 2, ok, 1, 8, 5120, 644, ok, NULL, NULL) == 1 and "dtype" in _err(L)
    assert L.qsa_indexer_project(ok, 1, ok, 1, 8, 5121, 644, ok, NULL, NULL) == 2
    assert L.qsa_indexer_project(NULL, 1, ok, 1, 8, 5120, 644, ok, NULL, NULL) == 1 and "null" in _err(L)
    assert L.qsa_indexer_project(ctypes.c_void_p(0x2004), 1, ok, 1, 8, 5120, 644, ok, NULL, NULL) == 1
    assert L.qsa_indexer_project(NULL, 1, NULL, 1, 0, 5120, 644, NULL, NULL, NULL) == 0
    assert L.qsa_indexer_project_workspace_size(8192, 5120, 644) == 0
    # (k_tok, tok_stride, n, g_req, g_id, wphi, bias, D_I, pages, k_dt, num_pages, pt, pt_rows, pt_stride, st, s)
    assert L.qsa_compress_keys(ok, 128, 4, NULL, ok, ok, NULL, 96, ok, 0, 4, ok, 1, 4, NULL, NULL) == 2
    assert L.qsa_compress_keys(ok, 64, 4, NULL, ok, ok, NULL, 128, ok, 0, 4, ok, 1, 4, NULL, NULL) == 1
    assert "tok_stride" in _err(L)
    assert L.qsa_compress_keys(ok, 128, 4, NULL, ok, ok, NULL, 128, ok, 2, 4, ok, 1, 4, NULL, NULL) == 1
    assert L.qsa_compress_keys(ok, 128, 4, NULL, NULL, ok, NULL, 128, ok, 0, 4, ok, 1, 4, NULL, NULL) == 1
    assert L.qsa_compress_keys(NULL, 128, 0, NULL, NULL, NULL, NULL, 128, NULL, 0, 4, NULL, 1, 4, NULL, NULL) == 0
    assert L.qsa_compress_keys_workspace_size(2048, 128) == 0


def test_seq_len_threshold_resolution(L):
    """TensorRT-LLM's rule: unset -> the token budget (4 tokens per group of
    the budget); an explicit value below the budget is raised to it."""
    assert L.qsa_seq_len_threshold(0, 512) == 2048
    assert L.qsa_seq_len_threshold(-5, 1024) == 4096
    assert L.qsa_seq_len_threshold(100, 512) == 2048
    assert L.qsa_seq_len_threshold(10000, 512) == 10000
    assert L.qsa_dense_select(NULL, 0, 100, NULL, NULL, 16, NULL, NULL) == 0
    assert L.qsa_dense_select(NULL, 2, 100, NULL, NULL, 16, NULL, NULL) == 1 and "null" in _err(L)
