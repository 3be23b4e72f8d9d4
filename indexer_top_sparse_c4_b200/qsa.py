"""Thin ctypes binding of libqsa.so (include/qsa.h).

Same names as the C entry points.  Each function only turns torch tensors
into pointers, dtypes and sizes and calls the library on the current CUDA
stream; every step of the computation runs in the library's kernels.  There
is no fallback: if libqsa.so is missing or a call fails, an exception is
raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqsa.so")

(QSA_OK, QSA_ERR_INVALID_ARG, QSA_ERR_UNSUPPORTED, QSA_ERR_WORKSPACE, QSA_ERR_CUDA,
 QSA_ERR_DEVICE_INDEX, QSA_ERR_TIMEOUT) = range(7)
QSA_F32, QSA_BF16, QSA_FP8_E4M3 = 0, 1, 2
QSA_DEV_BAD_PAGE, QSA_DEV_BAD_TOKEN, QSA_DEV_BAD_GROUP, QSA_DEV_ROW_RANGE = 1, 2, 4, 8
QSA_DEV_BAD_REQUEST, QSA_DEV_TIMEOUT = 16, 32
QSA_PREFIX_HIST_BINS = 4096

ENTRY_POINTS = (
    "qsa_indexer_project_workspace_size", "qsa_indexer_project", "qsa_compress_keys_workspace_size",
    "qsa_compress_keys",
    "qsa_index_scores_workspace_size", "qsa_index_scores", "qsa_topk_groups_workspace_size",
    "qsa_topk_groups", "qsa_topk_groups_gvr", "qsa_expand_select_workspace_size", "qsa_expand_select", "qsa_topk_expand",
    "qsa_seq_len_threshold", "qsa_dense_select",
    "qsa_sparse_attn_decode_workspace_size", "qsa_sparse_attn_decode",
    "qsa_sparse_attn_decode_sel_workspace_size", "qsa_sparse_attn_decode_sel",
    "qsa_sparse_attn_prefill_workspace_size", "qsa_sparse_attn_prefill", "qsa_get_device_status",
    "qsa_dcp_shard_positions", "qsa_dcp_candidates", "qsa_dcp_merge_topk", "qsa_dcp_expand",
    "qsa_dcp_merge_attn", "qsa_selftest_bounded_wait",
    "qsa_last_error_string", "qsa_status_name", "qsa_abi_version",
)


class QSAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_status_name(status)}: {msg}")
        self.status = status


_lib: Optional[ctypes.CDLL] = None


_binding = None   # a _Recorder while bind() runs a wrapper


class _Recorder:
    """Stands in for the library while bind() runs a wrapper: the launching
    calls are recorded with their converted arguments (and report QSA_OK),
    everything else (size queries, names) goes to the library."""

    def __init__(self, real):
        self.real, self.calls = real, []

    def __getattr__(self, name):
        fn = getattr(self.real, name)
        if name.endswith("_workspace_size") or name in ("qsa_last_error_string", "qsa_status_name",
                                                        "qsa_abi_version", "qsa_seq_len_threshold"):
            return fn

        def record(*args):
            self.calls.append((fn, args))
            return QSA_OK
        return record


def bind(fn, *args, **kwargs):
    """The libqsa calls that ``fn(*args, **kwargs)`` makes, with their
    ctypes arguments built once: returns a zero-argument callable that only
    crosses into C, for host-bound loops.  The tensors and the stream the
    calls name are fixed at binding: they must stay allocated and in place
    (bind again after replacing one), and ``stream=None`` means the stream
    current now.  Bind from one thread at a time: while ``fn`` runs, lib()
    hands out the recorder."""
    global _binding
    rec = _Recorder(lib())
    _binding = rec
    try:
        fn(*args, **kwargs)
    finally:
        _binding = None
    calls = tuple(rec.calls)

    def call():
        for f, a in calls:
            _check(f(*a))
    return call


def lib() -> ctypes.CDLL:
    """Load libqsa.so (built in-tree by ``python -m indexer_top_sparse_c4_b200.build``)."""
    global _lib
    if _binding is not None:
        return _binding
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m indexer_top_sparse_c4_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, U = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.qsa_indexer_project_workspace_size.argtypes = [I, I, I]
    L.qsa_indexer_project_workspace_size.restype = U
    L.qsa_indexer_project.argtypes = [P, I, P, I, I, I, I, P, P, P]
    L.qsa_indexer_project.restype = I
    L.qsa_compress_keys_workspace_size.argtypes = [I, I]
    L.qsa_compress_keys_workspace_size.restype = U
    L.qsa_compress_keys.argtypes = [P, I, I, P, P, P, P, I, P, I, I, P, I, I, P, P]
    L.qsa_compress_keys.restype = I
    L.qsa_seq_len_threshold.argtypes = [I, I]
    L.qsa_seq_len_threshold.restype = I
    L.qsa_dense_select.argtypes = [P, I, I, P, P, I, P, P]
    L.qsa_dense_select.restype = I
    L.qsa_topk_groups_gvr.argtypes = [P, I, P, I, I, P, P, P, P, P]
    L.qsa_topk_groups_gvr.restype = I
    L.qsa_dcp_shard_positions.argtypes = [P, I, I, I, P, P]
    L.qsa_dcp_candidates.argtypes = [P, I, P, P, I, I, I, P, P, P, P]
    L.qsa_dcp_merge_topk.argtypes = [P, P, I, I, I, P, P, P]
    L.qsa_dcp_expand.argtypes = [P, P, I, P, I, I, I, P, P, I, P, P]
    L.qsa_dcp_merge_attn.argtypes = [P, P, I, I, I, I, P, I, P, P]
    for name in ("qsa_dcp_shard_positions", "qsa_dcp_candidates", "qsa_dcp_merge_topk", "qsa_dcp_expand",
                 "qsa_dcp_merge_attn"):
        getattr(L, name).restype = I
    L.qsa_index_scores_workspace_size.argtypes = [I, I, I, I]
    L.qsa_index_scores_workspace_size.restype = U
    L.qsa_expand_select_workspace_size.argtypes = [I, I, I]
    L.qsa_expand_select_workspace_size.restype = U
    L.qsa_sparse_attn_prefill_workspace_size.argtypes = [I, I, I, I, I, I]
    L.qsa_sparse_attn_prefill_workspace_size.restype = U
    L.qsa_get_device_status.argtypes = [P, P, I, P]
    L.qsa_get_device_status.restype = I
    L.qsa_selftest_bounded_wait.argtypes = [ctypes.c_uint32, P, P, P]
    L.qsa_selftest_bounded_wait.restype = I
    L.qsa_index_scores.argtypes = [P, I, P, P, I, I, P, I, I, P, P, I, I, I, P, I, P, P, P]
    L.qsa_topk_groups_workspace_size.argtypes = [I, I, I]
    L.qsa_topk_groups_workspace_size.restype = U
    L.qsa_topk_groups.argtypes = [P, I, P, P, I, I, P, P, P, U, P, P]
    L.qsa_expand_select.argtypes = [P, P, I, P, P, I, P, P, I, P, P]
    L.qsa_topk_expand.argtypes = [P, I, P, P, I, I, P, P, P, P, I, P, P]
    L.qsa_sparse_attn_decode_workspace_size.argtypes = [I, I, I, I, I, I]
    L.qsa_sparse_attn_decode_workspace_size.restype = U
    L.qsa_sparse_attn_decode.argtypes = [P, I, P, P, I, F, F, I, P, I, I, P, P, P, I, I, I, I, I,
                                         F, P, I, P, P, U, P, P]
    L.qsa_sparse_attn_prefill.argtypes = [P, I, P, P, I, F, F, I, P, I, I, P, P, P, I, I, I, I, I,
                                          F, P, I, P, P, P]
    L.qsa_sparse_attn_decode_sel_workspace_size.argtypes = [I, I, I, I, I, I]
    L.qsa_sparse_attn_decode_sel_workspace_size.restype = U
    L.qsa_sparse_attn_decode_sel.argtypes = [P, I, P, P, I, F, F, I, P, I, I, P, P, P, I, P, P, I, I, I, I, I,
                                             F, P, I, P, P, U, P, P]
    L.qsa_sparse_attn_decode_sel.restype = I
    for name in ("qsa_index_scores", "qsa_topk_groups", "qsa_expand_select", "qsa_topk_expand",
                 "qsa_sparse_attn_decode", "qsa_sparse_attn_prefill"):
        getattr(L, name).restype = I
    L.qsa_last_error_string.restype = ctypes.c_char_p
    L.qsa_status_name.restype = ctypes.c_char_p
    L.qsa_status_name.argtypes = [I]
    L.qsa_abi_version.restype = I
    _lib = L
    return L


def _status_name(s: int) -> str:
    try:
        return lib().qsa_status_name(s).decode()
    except Exception:
        return f"status {s}"


def _check(status: int):
    if status != QSA_OK:
        raise QSAError(status, lib().qsa_last_error_string().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("libqsa takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return QSA_F32
    if t.dtype == torch.bfloat16:
        return QSA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return QSA_FP8_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def qsa_index_scores(q_idx, w_idx, k_idx_pages, page_table, q_pos, scores, q_req=None,
                     dev_status=None, stream=None, prefix_hist=None):
    """prefix_hist: optional int32/uint32 [T, QSA_PREFIX_HIST_BINS], zero on
    entry; receives the row's 12-bit key-prefix counts (see qsa.h)."""
    T, H_I, D_I = q_idx.shape
    _check(lib().qsa_index_scores(
        _ptr(q_idx), _dt(q_idx), _ptr(w_idx), _ptr(k_idx_pages), _dt(k_idx_pages),
        k_idx_pages.shape[0], _ptr(page_table), page_table.shape[0], page_table.shape[1],
        _ptr(q_req), _ptr(q_pos),
        T, H_I, D_I, _ptr(scores), scores.shape[1], _ptr(prefix_hist), _ptr(dev_status),
        _stream(stream)))
    return scores


def qsa_indexer_project(x, w, y, dev_status=None, stream=None):
    """y [T, N] float32 = x [T, H] . w [N, H]^T (x and w float32 or bfloat16)."""
    T, H = x.shape
    N, H2 = w.shape
    if H2 != H or tuple(y.shape) != (T, N) or y.dtype != torch.float32:
        raise ValueError("shapes: x [T, H], w [N, H], y [T, N] float32")
    _check(lib().qsa_indexer_project(_ptr(x), _dt(x), _ptr(w), _dt(w), T, H, N, _ptr(y), _ptr(dev_status),
                                     _stream(stream)))
    return y


def qsa_compress_keys(k_tok, g_id, wphi, k_idx_pages, page_table, g_req=None, bias=None, dev_status=None,
                      stream=None):
    """The C4 compressed-key write.  k_tok: float32 [4 * n, D_I] token keys,
    four consecutive rows per completed group; its rows may be strided (a
    column slice of qsa_indexer_project's output) but each row contiguous."""
    if k_tok.dtype != torch.float32 or k_tok.dim() != 2 or k_tok.stride(1) != 1:
        raise ValueError("k_tok must be float32 [4 * n, D_I] with contiguous rows")
    rows, D_I = k_tok.shape
    n = g_id.numel()
    if rows != 4 * n:
        raise ValueError("k_tok must hold four token rows per group")
    _check(lib().qsa_compress_keys(
        ctypes.c_void_p(k_tok.data_ptr()), k_tok.stride(0), n, _ptr(g_req), _ptr(g_id), _ptr(wphi), _ptr(bias),
        D_I, _ptr(k_idx_pages), _dt(k_idx_pages), k_idx_pages.shape[0], _ptr(page_table), page_table.shape[0],
        page_table.shape[1], _ptr(dev_status), _stream(stream)))
    return k_idx_pages


def qsa_index_scores_workspace_size(T, H_I, D_I, score_stride) -> int:
    return int(lib().qsa_index_scores_workspace_size(T, H_I, D_I, score_stride))


def qsa_expand_select_workspace_size(T, K, W) -> int:
    return int(lib().qsa_expand_select_workspace_size(T, K, W))


def qsa_sparse_attn_prefill_workspace_size(T, Hq, Hkv, D, W, kv_dtype=QSA_BF16) -> int:
    if isinstance(kv_dtype, torch.dtype):
        kv_dtype = _dt(torch.empty(0, dtype=kv_dtype))
    return int(lib().qsa_sparse_attn_prefill_workspace_size(T, Hq, Hkv, D, W, kv_dtype))


def qsa_selftest_bounded_wait(limit_us, dev_status, report, stream=None):
    """Run the bounded-wait self-test (a wait on a barrier nothing arrives
    at, with a limit of limit_us): report is int32 [6] on the device."""
    if report.numel() < 6 or report.dtype != torch.int32:
        raise ValueError("report must be int32 with at least 6 elements")
    _check(lib().qsa_selftest_bounded_wait(int(limit_us), _ptr(dev_status), _ptr(report), _stream(stream)))
    return report


def qsa_get_device_status(dev_status, clear=False, stream=None):
    """Read the caller's device status word on the host (synchronises the
    stream).  Returns (status, bits): QSA_OK, QSA_ERR_DEVICE_INDEX or
    QSA_ERR_TIMEOUT and the raw word.  Other codes raise QSAError."""
    bits = ctypes.c_uint32(0)
    st = lib().qsa_get_device_status(_ptr(dev_status), ctypes.byref(bits), 1 if clear else 0,
                                     _stream(stream))
    if st not in (QSA_OK, QSA_ERR_DEVICE_INDEX, QSA_ERR_TIMEOUT):
        raise QSAError(st, lib().qsa_last_error_string().decode())
    return st, int(bits.value)


def qsa_topk_groups_workspace_size(T, K, score_stride) -> int:
    return int(lib().qsa_topk_groups_workspace_size(T, K, score_stride))


def qsa_topk_groups(scores, q_pos, K, sel, n_sel, workspace=None, dev_status=None, stream=None,
                    prefix_hist=None):
    T = scores.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().qsa_topk_groups(
        _ptr(scores), scores.shape[1], _ptr(prefix_hist), _ptr(q_pos), T, K, _ptr(sel), _ptr(n_sel),
        _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream)))
    return sel, n_sel


def qsa_seq_len_threshold(requested, K) -> int:
    """Tokens at or below which a sequence takes dense attention (None or
    <= 0: the token budget 4*K; never below it)."""
    return int(lib().qsa_seq_len_threshold(int(requested or 0), int(K)))


def qsa_dense_select(q_pos, threshold, tok, n_tok, dev_status=None, stream=None):
    T, W = tok.shape
    _check(lib().qsa_dense_select(_ptr(q_pos), T, int(threshold), _ptr(tok), _ptr(n_tok), W, _ptr(dev_status),
                                  _stream(stream)))
    return tok, n_tok


def qsa_topk_groups_gvr(scores, q_pos, K, sel, n_sel, path=None, dev_status=None, stream=None):
    """The guess-verify-refine Top-K (same result as qsa_topk_groups);
    path: optional int32 [T] receiving how each row was selected."""
    T = scores.shape[0]
    _check(lib().qsa_topk_groups_gvr(_ptr(scores), scores.shape[1], _ptr(q_pos), T, K, _ptr(sel), _ptr(n_sel),
                                     _ptr(path), _ptr(dev_status), _stream(stream)))
    return sel, n_sel


def qsa_expand_select(sel, n_sel, q_pos, tok, n_tok, capture_pos=None, dev_status=None, stream=None):
    T, K = sel.shape
    _check(lib().qsa_expand_select(
        _ptr(sel), _ptr(n_sel), K, _ptr(q_pos), _ptr(capture_pos), T, _ptr(tok), _ptr(n_tok),
        tok.shape[1], _ptr(dev_status), _stream(stream)))
    return tok, n_tok


def qsa_topk_expand(scores, q_pos, K, sel, n_sel, tok, n_tok, dev_status=None, stream=None,
                    prefix_hist=None):
    """Top-K and expansion in one launch (rows without an MTP capture)."""
    T, score_stride = scores.shape
    _check(lib().qsa_topk_expand(
        _ptr(scores), score_stride, _ptr(prefix_hist), _ptr(q_pos), T, K, _ptr(sel), _ptr(n_sel),
        _ptr(tok), _ptr(n_tok), tok.shape[1], _ptr(dev_status), _stream(stream)))
    return sel, n_sel, tok, n_tok


def qsa_sparse_attn_decode_workspace_size(T, Hq, Hkv, D, W, kv_dtype=QSA_FP8_E4M3) -> int:
    """Bytes of workspace qsa_sparse_attn_decode needs; kv_dtype is a QSA_*
    code or a torch dtype of the KV cache."""
    if isinstance(kv_dtype, torch.dtype):
        kv_dtype = _dt(torch.empty(0, dtype=kv_dtype))
    return int(lib().qsa_sparse_attn_decode_workspace_size(T, Hq, Hkv, D, W, kv_dtype))


def _attn_args(q, k_pages, v_pages, page_table, tok, n_tok, out, k_scale, v_scale, q_req,
               sm_scale, lse):
    T, Hq, D = q.shape
    num_pages, _, Hkv, _ = k_pages.shape
    return [_ptr(q), _dt(q), _ptr(k_pages), _ptr(v_pages), _dt(k_pages), float(k_scale),
            float(v_scale), num_pages, _ptr(page_table), page_table.shape[0], page_table.shape[1],
            _ptr(q_req),
            _ptr(tok), _ptr(n_tok), tok.shape[1], T, Hq, Hkv, D, float(sm_scale), _ptr(out),
            _dt(out), _ptr(lse)]


def qsa_sparse_attn_decode(q, k_pages, v_pages, page_table, tok, n_tok, out, workspace=None,
                           k_scale=1.0, v_scale=1.0, q_req=None, sm_scale=0.0, lse=None,
                           dev_status=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = _attn_args(q, k_pages, v_pages, page_table, tok, n_tok, out, k_scale, v_scale, q_req,
                      sm_scale, lse)
    _check(lib().qsa_sparse_attn_decode(*args, _ptr(workspace), ws_bytes, _ptr(dev_status),
                                        _stream(stream)))
    return out


def qsa_sparse_attn_decode_sel_workspace_size(T, Hq, Hkv, D, W, kv_dtype=QSA_BF16) -> int:
    if isinstance(kv_dtype, torch.dtype):
        kv_dtype = _dt(torch.empty(0, dtype=kv_dtype))
    return int(lib().qsa_sparse_attn_decode_sel_workspace_size(T, Hq, Hkv, D, W, kv_dtype))


def qsa_sparse_attn_decode_sel(q, k_pages, v_pages, page_table, sel, n_sel, q_pos, W, out, workspace=None,
                               capture_pos=None, k_scale=1.0, v_scale=1.0, q_req=None, sm_scale=0.0, lse=None,
                               dev_status=None, stream=None):
    """Stages 3 and 4 in one call: the decode attention over the tokens the
    selection sel [T, K] / n_sel [T] expands to (plus 4*c(p0) .. p), W wide."""
    T, Hq, D = q.shape
    num_pages, _, Hkv, _ = k_pages.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().qsa_sparse_attn_decode_sel(
        _ptr(q), _dt(q), _ptr(k_pages), _ptr(v_pages), _dt(k_pages), float(k_scale), float(v_scale), num_pages,
        _ptr(page_table), page_table.shape[0], page_table.shape[1], _ptr(q_req), _ptr(sel), _ptr(n_sel),
        sel.shape[1], _ptr(q_pos), _ptr(capture_pos), int(W), T, Hq, Hkv, D, float(sm_scale), _ptr(out), _dt(out),
        _ptr(lse), _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream)))
    return out


def qsa_sparse_attn_prefill(q, k_pages, v_pages, page_table, tok, n_tok, out, k_scale=1.0,
                            v_scale=1.0, q_req=None, sm_scale=0.0, lse=None, dev_status=None,
                            stream=None):
    args = _attn_args(q, k_pages, v_pages, page_table, tok, n_tok, out, k_scale, v_scale, q_req,
                      sm_scale, lse)
    _check(lib().qsa_sparse_attn_prefill(*args, _ptr(dev_status), _stream(stream)))
    return out


def qsa_last_error_string() -> str:
    return lib().qsa_last_error_string().decode()


def qsa_abi_version() -> int:
    return int(lib().qsa_abi_version())


def qsa_sparse_attn_decode_noalloc(q, k_pages, v_pages, page_table, tok, n_tok, out, k_scale=1.0,
                                   v_scale=1.0, q_req=None, sm_scale=0.0, lse=None,
                                   dev_status=None, stream=None):
    """qsa_sparse_attn_decode without a workspace: for callers that cannot
    allocate device memory.  The library's own fixed scratch buffer is used
    (QSA_DECODE_NOALLOC_SCRATCH_BYTES per device); larger shapes raise
    QSAError(QSA_ERR_WORKSPACE).  Calls that overlap on the GPU share that
    buffer and must not run concurrently."""
    fn = lib().qsa_sparse_attn_decode_noalloc
    if fn.argtypes is None:
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        fn.argtypes = [P, I, P, P, I, F, F, I, P, I, I, P, P, P, I, I, I, I, I, F, P, I, P, P, P]
        fn.restype = I
    args = _attn_args(q, k_pages, v_pages, page_table, tok, n_tok, out, k_scale, v_scale, q_req,
                      sm_scale, lse)
    _check(fn(*args, _ptr(dev_status), _stream(stream)))
    return out


# ---- sequence-sharded decode ---------------------------------------------------------

def qsa_dcp_shard_positions(q_pos, g_lo, g_hi, q_pos_local, stream=None):
    _check(lib().qsa_dcp_shard_positions(_ptr(q_pos), q_pos.numel(), g_lo, g_hi, _ptr(q_pos_local),
                                         _stream(stream)))
    return q_pos_local


def qsa_dcp_candidates(scores, sel, n_sel, g_lo, cand_score, cand_id, dev_status=None, stream=None):
    T, K = sel.shape
    _check(lib().qsa_dcp_candidates(_ptr(scores), scores.shape[1], _ptr(sel), _ptr(n_sel), T, K, g_lo,
                                    _ptr(cand_score), _ptr(cand_id), _ptr(dev_status), _stream(stream)))
    return cand_score, cand_id


def qsa_dcp_merge_topk(cand_score, cand_id, sel, n_sel, stream=None):
    """cand_score / cand_id [R, T, K] -> sel [T, K], n_sel [T]."""
    R, T, K = cand_id.shape
    _check(lib().qsa_dcp_merge_topk(_ptr(cand_score), _ptr(cand_id), R, T, K, _ptr(sel), _ptr(n_sel),
                                    _stream(stream)))
    return sel, n_sel


def qsa_dcp_expand(sel, n_sel, q_pos, g_lo, g_hi, tok, n_tok, dev_status=None, stream=None):
    T, K = sel.shape
    _check(lib().qsa_dcp_expand(_ptr(sel), _ptr(n_sel), K, _ptr(q_pos), T, g_lo, g_hi, _ptr(tok), _ptr(n_tok),
                                tok.shape[1], _ptr(dev_status), _stream(stream)))
    return tok, n_tok


def qsa_dcp_merge_attn(o_parts, lse_parts, out, lse=None, stream=None):
    """o_parts [R, T, Hq, D] float32, lse_parts [R, T, Hq] -> out [T, Hq, D], lse [T, Hq]."""
    R, T, Hq, D = o_parts.shape
    _check(lib().qsa_dcp_merge_attn(_ptr(o_parts), _ptr(lse_parts), R, T, Hq, D, _ptr(out), _dt(out), _ptr(lse),
                                    _stream(stream)))
    return out
