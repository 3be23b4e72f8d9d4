"""CPU oracle for the QSA hot path (indexer scores -> exact Top-K -> expand -> attention).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product library (``libqsa.so``) and its binding never touch it;
the two share no code.

The arithmetic lives in ``qsa_oracle.c`` (plain C, double-precision
accumulation, its own BF16 / FP8-E4M3FN decoders).  This module only builds
that file with gcc and marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libqsa_oracle.so")

F32, BF16, FP8_E4M3 = 0, 1, 2
PAGE_TOKENS = 64
GROUP_TOKENS = 4
PAGE_GROUPS = PAGE_TOKENS // GROUP_TOKENS


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libqsa_oracle.so`` (gcc, -O2, OpenMP)."""
    hdr = os.path.join(_HERE, "qsa_oracle.h")
    if not force and os.path.exists(_LIB_PATH):
        newest = max(os.path.getmtime(_SRC), os.path.getmtime(hdr))
        if os.path.getmtime(_LIB_PATH) >= newest:
            return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P, I, L, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_float
        _lib.orc_bf16_to_f64.restype = ctypes.c_double
        _lib.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
        _lib.orc_e4m3_to_f64.restype = ctypes.c_double
        _lib.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        _lib.orc_index_scores.restype = L
        _lib.orc_index_scores.argtypes = [P, I, P, P, I, I, P, I, P, P, I, I, I, P, I]
        _lib.orc_topk_groups.restype = L
        _lib.orc_topk_groups.argtypes = [P, I, P, I, I, P, P]
        _lib.orc_expand_select.restype = L
        _lib.orc_expand_select.argtypes = [P, P, I, P, P, I, P, P, I]
        _lib.orc_sparse_attn.restype = L
        _lib.orc_sparse_attn.argtypes = [P, I, P, P, I, F, F, I, P, I, P, P, P, I, I, I,
                                         I, I, F, P, P]
        _lib.orc_indexer_project.restype = L
        _lib.orc_indexer_project.argtypes = [P, I, P, I, I, I, I, P]
        _lib.orc_compress_keys.restype = L
        _lib.orc_compress_keys.argtypes = [P, I, P, P, P, P, I, P, I, I, P, I, I]
        _lib.orc_threads_for.restype = I
        _lib.orc_threads_for.argtypes = [I]
        _lib.orc_set_max_threads.restype = None
        _lib.orc_set_max_threads.argtypes = [I]
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dt_of(a: np.ndarray, fp8: bool = False) -> int:
    """float32 -> F32, uint16 (bf16 bit patterns) -> BF16, uint8 (E4M3 codes) -> FP8."""
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.uint8:
        return FP8_E4M3
    raise TypeError(f"unsupported oracle input dtype {a.dtype}")


def bf16_to_f64(bits: int) -> float:
    return lib().orc_bf16_to_f64(bits)


def e4m3_to_f64(code: int) -> float:
    return lib().orc_e4m3_to_f64(code)


def threads_for(T: int) -> int:
    return lib().orc_threads_for(T)


def set_max_threads(n: int) -> None:
    """Cap the OpenMP threads of the oracle's loops over query tokens."""
    lib().orc_set_max_threads(int(n))


def index_scores(q_idx, w_idx, k_idx_pages, page_table, q_pos, q_req=None, score_stride=None):
    """Stage 1.  Returns (scores [T, score_stride] float32, skipped-group count)."""
    q_idx = np.ascontiguousarray(q_idx)
    k_idx_pages = np.ascontiguousarray(k_idx_pages)
    T, H_I, D_I = q_idx.shape
    num_pages = k_idx_pages.shape[0]
    assert k_idx_pages.shape[1:] == (PAGE_GROUPS, D_I)
    pt = _c(page_table, np.int32)
    q_pos = _c(q_pos, np.int32)
    if score_stride is None:
        score_stride = int(max(1, (int(q_pos.max()) // GROUP_TOKENS) if T else 1))
    scores = np.empty((T, score_stride), np.float32)
    w = _c(w_idx, np.float32)
    qr = None if q_req is None else _c(q_req, np.int32)
    rc = lib().orc_index_scores(_ptr(q_idx), _dt_of(q_idx), _ptr(w), _ptr(k_idx_pages),
                                _dt_of(k_idx_pages), num_pages, _ptr(pt), pt.shape[1],
                                _ptr(qr), _ptr(q_pos), T, H_I, D_I, _ptr(scores), score_stride)
    if rc < 0:
        raise ValueError(f"orc_index_scores failed ({rc})")
    return scores, int(rc)


def topk_groups(scores, q_pos, K):
    """Stage 2.  Returns (sel [T,K] int32 ascending with -1 padding, n_sel [T])."""
    scores = _c(scores, np.float32)
    q_pos = _c(q_pos, np.int32)
    T = scores.shape[0]
    sel = np.empty((T, K), np.int32)
    n_sel = np.empty((T,), np.int32)
    rc = lib().orc_topk_groups(_ptr(scores), scores.shape[1], _ptr(q_pos), T, K, _ptr(sel), _ptr(n_sel))
    if rc < 0:
        raise ValueError(f"orc_topk_groups failed ({rc})")
    return sel, n_sel


def expand_select(sel, n_sel, q_pos, W, capture_pos=None):
    """Stage 3.  Returns (tok [T,W] int32, n_tok [T], count of invalid sel entries)."""
    sel = _c(sel, np.int32)
    n_sel = _c(n_sel, np.int32)
    q_pos = _c(q_pos, np.int32)
    T, K = sel.shape
    cap = None if capture_pos is None else _c(capture_pos, np.int32)
    tok = np.empty((T, W), np.int32)
    n_tok = np.empty((T,), np.int32)
    rc = lib().orc_expand_select(_ptr(sel), _ptr(n_sel), K, _ptr(q_pos), _ptr(cap), T,
                                 _ptr(tok), _ptr(n_tok), W)
    if rc < 0:
        raise ValueError(f"orc_expand_select failed ({rc})")
    return tok, n_tok, int(rc)


def sparse_attn(q, k_pages, v_pages, page_table, tok, n_tok, k_scale=1.0, v_scale=1.0,
                q_req=None, sm_scale=0.0):
    """Stage 4.  Returns (out [T,Hq,D] float64, lse [T,Hq] float64, skipped count)."""
    q = np.ascontiguousarray(q)
    k_pages = np.ascontiguousarray(k_pages)
    v_pages = np.ascontiguousarray(v_pages)
    T, Hq, D = q.shape
    num_pages, pg, Hkv, D2 = k_pages.shape
    assert pg == PAGE_TOKENS and D2 == D and v_pages.shape == k_pages.shape
    assert k_pages.dtype == v_pages.dtype
    pt = _c(page_table, np.int32)
    tok = _c(tok, np.int32)
    n_tok = _c(n_tok, np.int32)
    qr = None if q_req is None else _c(q_req, np.int32)
    out = np.empty((T, Hq, D), np.float64)
    lse = np.empty((T, Hq), np.float64)
    rc = lib().orc_sparse_attn(_ptr(q), _dt_of(q), _ptr(k_pages), _ptr(v_pages), _dt_of(k_pages),
                               float(k_scale), float(v_scale), num_pages, _ptr(pt), pt.shape[1],
                               _ptr(qr), _ptr(tok), _ptr(n_tok), tok.shape[1], T, Hq, Hkv, D,
                               float(sm_scale), _ptr(out), _ptr(lse))
    if rc < 0:
        raise ValueError(f"orc_sparse_attn failed ({rc})")
    return out, lse, int(rc)


def indexer_project(x, w):
    """Before stage 1: y [T,N] float32 = x [T,H] . w [N,H]^T (float32 or BF16
    bit patterns as uint16), accumulated in double."""
    x = np.ascontiguousarray(x)
    w = np.ascontiguousarray(w)
    T, H = x.shape
    N, H2 = w.shape
    assert H2 == H
    y = np.empty((T, N), np.float32)
    rc = lib().orc_indexer_project(_ptr(x), _dt_of(x), _ptr(w), _dt_of(w), T, H, N, _ptr(y))
    if rc < 0:
        raise ValueError(f"orc_indexer_project failed ({rc})")
    return y


def compress_keys(k_tok, g_id, wphi, k_idx_pages, page_table, g_req=None, bias=None):
    """Before stage 1: the C4 compressed-key write.  k_tok [n,4,D_I] float32
    token keys of n completed groups; writes each group's compressed key into
    k_idx_pages (float32, or uint16 BF16 bit patterns) IN PLACE through the
    page table.  Returns the count of skipped groups."""
    k_tok = _c(k_tok, np.float32)
    n, four, D_I = k_tok.shape
    assert four == GROUP_TOKENS
    assert k_idx_pages.flags.c_contiguous and k_idx_pages.shape[1:] == (PAGE_GROUPS, D_I)
    wphi = _c(wphi, np.float32)
    assert wphi.shape == (D_I, GROUP_TOKENS * D_I)
    b = None if bias is None else _c(bias, np.float32)
    pt = _c(page_table, np.int32)
    gid = _c(g_id, np.int32)
    gr = None if g_req is None else _c(g_req, np.int32)
    rc = lib().orc_compress_keys(_ptr(k_tok), n, _ptr(gr), _ptr(gid), _ptr(wphi), _ptr(b), D_I,
                                 _ptr(k_idx_pages), _dt_of(k_idx_pages), k_idx_pages.shape[0], _ptr(pt),
                                 pt.shape[0], pt.shape[1])
    if rc < 0:
        raise ValueError(f"orc_compress_keys failed ({rc})")
    return int(rc)


def qsa_step(q, q_idx, w_idx, k_idx_pages, k_pages, v_pages, page_table, q_pos, K,
             k_scale=1.0, v_scale=1.0, q_req=None, capture_pos=None, sm_scale=0.0):
    """All four stages chained, as the method defines them.  Returns a dict."""
    q_pos = _c(q_pos, np.int32)
    sel_pos = q_pos if capture_pos is None else _c(capture_pos, np.int32)
    stride = int(max(1, int(q_pos.max()) // GROUP_TOKENS))
    scores, _ = index_scores(q_idx, w_idx, k_idx_pages, page_table, sel_pos, q_req, stride)
    sel, n_sel = topk_groups(scores, sel_pos, K)
    W = 4 * K + 4 + (0 if capture_pos is None else 4 * int(
        (q_pos // 4 - sel_pos // 4).max(initial=0)))
    tok, n_tok, _ = expand_select(sel, n_sel, q_pos, W, capture_pos)
    out, lse, _ = sparse_attn(q, k_pages, v_pages, page_table, tok, n_tok, k_scale, v_scale,
                              q_req, sm_scale)
    return dict(scores=scores, sel=sel, n_sel=n_sel, tok=tok, n_tok=n_tok, out=out, lse=lse, W=W)
