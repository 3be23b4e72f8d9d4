"""Helpers shared by the GPU parity tests: tolerances, host copies in the
oracle's formats, compaction of the pages a selection touches."""
from __future__ import annotations

import numpy as np
import torch

# attention tolerances against the FP64 oracle (max-abs 2e-2 and mean-abs
# 2e-3 for BF16 / FP8 KV, the target stated for this path; rel-L2 as the
# Ascend article's operator tests use)
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
ATTN_REL_L2 = 8e-3
# indexer score tolerance, relative to the dot-product error scale
SCORE_REL = 1e-4


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def values_f64(a: np.ndarray) -> np.ndarray:
    """The stored values as float64: BF16 bit patterns (uint16, the host form
    of BF16 tensors) are widened to the floats they encode."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def score_bound(q_idx: np.ndarray, w_idx: np.ndarray, khat: np.ndarray, page_table: np.ndarray,
                q_req: np.ndarray, q_pos: np.ndarray, rows, stride: int) -> np.ndarray:
    """SCORE_REL * sum_h |w_h| sum_d |q_hd k_d| for every (row, group) in rows."""
    out = np.zeros((len(rows), stride))
    for i, t in enumerate(rows):
        c = min(int(q_pos[t]) // 4, stride)
        if c == 0:
            continue
        r = int(q_req[t]) if q_req is not None else t
        pages = page_table[r][: (c + 15) // 16]
        k = np.abs(values_f64(khat[pages].reshape(-1, khat.shape[-1])[:c]))
        q = np.abs(values_f64(q_idx[t]))                   # [H, D]
        out[i, :c] = (np.abs(values_f64(w_idx[t])) @ (q @ k.T)) * SCORE_REL
    return out


def compact_pages(k_pages: torch.Tensor, v_pages: torch.Tensor, page_table: torch.Tensor,
                  tok: np.ndarray, n_tok: np.ndarray, req: np.ndarray):
    """Copy to the host only the pages the token lists touch, with a page table
    that maps the same logical pages onto the compact copy."""
    pt = page_table.cpu().numpy()
    B, P = pt.shape
    used = np.zeros((B, P), bool)
    for i in range(tok.shape[0]):
        row = tok[i, : n_tok[i]]
        row = row[(row >= 0) & (row < P * 64)]
        used[int(req[i]), row // 64] = True
    new_pt = np.full((B, P), 0, np.int32)
    phys = []
    for r in range(B):
        for lp in np.nonzero(used[r])[0]:
            new_pt[r, lp] = len(phys)
            phys.append(pt[r, lp])
    phys_t = torch.as_tensor(np.array(phys if phys else [0], np.int64), device=k_pages.device)
    kc = host(k_pages.index_select(0, phys_t))
    vc = host(v_pages.index_select(0, phys_t))
    return kc, vc, new_pt


def attn_errors(gpu: np.ndarray, ref: np.ndarray):
    d = np.abs(gpu.astype(np.float64) - ref)
    rel = np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30)
    return float(d.max(initial=0.0)), float(d.mean() if d.size else 0.0), float(rel)


def out_as_f64(out: torch.Tensor) -> np.ndarray:
    return out.detach().float().cpu().numpy().astype(np.float64)
