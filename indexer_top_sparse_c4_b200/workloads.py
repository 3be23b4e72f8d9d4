"""Seeded synthetic inputs for the QSA hot path.

This module only draws random numbers and lays them out in the storage formats
the library reads (paged KV cache, paged compressed indexer keys, page tables,
query positions).  It holds none of the method's arithmetic, so both the CUDA
path and the CPU oracle can be fed from it.

Storage formats (shared by the library and the oracle):
  * KV pages      [num_pages, 64, Hkv, D]   float32 | bfloat16 | uint8 (E4M3FN codes)
  * indexer keys  [num_pages, 16, D_I]      float32 (one key per 4-token group;
                                             a 64-token page holds 16 groups and
                                             shares the KV page table)
  * page table    [B, pages_per_request]    int32 physical page ids
  * q [T,Hq,D], q_idx [T,H_I,D_I], w_idx [T,H_I], q_req [T], q_pos [T]

Score distributions for the indexer keys:
  normal  -- khat ~ N(0,1)
  peaked  -- 5% of groups (seeded Bernoulli) get khat += b, b the minimum-norm
             vector with q_h . b = 3 |q_h| for every indexer head of the
             request's decode query, i.e. a +3 sigma shift of every head's dot
  ties    -- q_h = e_0, w_h = 1/H_I, khat[:,0] = level in {0..15}: every score
             is exactly its level, so the ranking is decided by the group-index
             tie-break
  dyadic  -- q_idx, khat on the grid (1/8)Z within [-4,4] and w on (1/16)Z in
             [0,1]: every summation order yields the same float32 score
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

PAGE_TOKENS = 64
GROUP_TOKENS = 4
PAGE_GROUPS = PAGE_TOKENS // GROUP_TOKENS
FP8_MAX = 448.0


@dataclasses.dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    H_I: int
    D_I: int
    K: int                      # budget in groups
    W: int                      # width of the expanded token list
    kv_dtype: str               # "f32" | "bf16" | "fp8"
    q_dtype: str                # "f32" | "bf16"
    q: torch.Tensor
    q_idx: torch.Tensor
    w_idx: torch.Tensor
    k_idx_pages: torch.Tensor
    k_pages: torch.Tensor
    v_pages: torch.Tensor
    k_scale: float
    v_scale: float
    page_table: torch.Tensor
    q_req: torch.Tensor
    q_pos: torch.Tensor
    capture_pos: Optional[torch.Tensor] = None
    dist: str = "normal"
    seed: int = 0

    @property
    def T(self) -> int:
        return self.q.shape[0]

    @property
    def num_pages(self) -> int:
        return self.k_pages.shape[0]

    @property
    def score_stride(self) -> int:
        return max(1, int(self.q_pos.max().item()) // GROUP_TOKENS)

    def to(self, device) -> "Workload":
        kw = {}
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            kw[f.name] = v.to(device) if isinstance(v, torch.Tensor) else v
        return Workload(**kw)

    def numpy(self) -> dict:
        """Host copies in the oracle's input formats (bf16 as uint16 bit patterns)."""
        def n(t):
            if t is None:
                return None
            t = t.detach().cpu().contiguous()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view("uint16")
            return t.numpy()
        return {f.name: n(getattr(self, f.name)) for f in dataclasses.fields(self)
                if f.type in ("torch.Tensor", "Optional[torch.Tensor]")}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _store(x: torch.Tensor, dtype: str):
    """Store float32 values in a KV / query storage format.  FP8 uses one
    per-tensor scale, amax/448, and round-to-nearest-even codes."""
    if dtype == "f32":
        return x.contiguous(), 1.0
    if dtype == "bf16":
        return x.to(torch.bfloat16).contiguous(), 1.0
    if dtype == "fp8":
        amax = float(x.abs().max().item())
        scale = amax / FP8_MAX if amax > 0 else 1.0
        scale = float(torch.tensor(scale, dtype=torch.float32).item())   # an FP32 scale
        codes = (x / scale).clamp_(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn)
        return codes.view(torch.uint8).contiguous(), scale
    raise ValueError(dtype)


def page_table_for(B: int, pages_per_req: int, kind: str, g, device) -> torch.Tensor:
    """identity: request r owns pages r*P..r*P+P-1 in order; perm: a seeded
    random permutation of all B*P physical pages."""
    total = B * pages_per_req
    if kind == "identity":
        ids = torch.arange(total, device=device, dtype=torch.int64)
    elif kind == "perm":
        ids = torch.randperm(total, generator=g, device=device)
    else:
        raise ValueError(kind)
    return ids.to(torch.int32).view(B, pages_per_req).contiguous()


def _indexer_inputs(T, H_I, D_I, num_pages, dist, g, device, q_req, B):
    """q_idx [T,H_I,D_I], w_idx [T,H_I], khat pages [num_pages,16,D_I]."""
    if dist == "ties":
        q_idx = torch.zeros((T, H_I, D_I), device=device)
        q_idx[:, :, 0] = 1.0
        w_idx = torch.full((T, H_I), 1.0 / H_I, device=device)
        khat = _randn((num_pages, PAGE_GROUPS, D_I), g, device)
        lv = torch.randint(0, 16, (num_pages, PAGE_GROUPS), generator=g, device=device)
        khat[:, :, 0] = lv.to(torch.float32)
        return q_idx, w_idx, khat
    q_idx = _randn((T, H_I, D_I), g, device)
    w_idx = torch.rand((T, H_I), generator=g, device=device, dtype=torch.float32)
    khat = _randn((num_pages, PAGE_GROUPS, D_I), g, device)
    if dist == "dyadic":
        q_idx = (q_idx * 8).round_().clamp_(-32, 32) / 8
        khat = (khat * 8).round_().clamp_(-32, 32) / 8
        w_idx = (w_idx * 16).round_() / 16
    elif dist == "peaked":
        pass  # bias is added per request by the caller (needs the page table)
    elif dist != "normal":
        raise ValueError(dist)
    return q_idx.contiguous(), w_idx.contiguous(), khat.contiguous()


def _add_peaks(khat, q_idx, page_table, q_req, g, device, frac=0.05, sigmas=3.0):
    """+3 sigma on every indexer head's dot for a seeded 5% of each request's
    groups; sigma_h = |q_h| is the spread of q_h . z for z ~ N(0, I)."""
    B, P = page_table.shape
    for r in range(B):
        rows = (q_req == r).nonzero().flatten()
        if rows.numel() == 0:
            continue
        Q = q_idx[int(rows[0])].double()                          # [H_I, D_I]
        target = sigmas * Q.norm(dim=1)                           # [H_I]
        b = (torch.linalg.pinv(Q) @ target).float()               # min-norm solution
        m = torch.rand((P * PAGE_GROUPS,), generator=g, device=device) < frac
        pages = page_table[r].long()
        view = khat[pages].view(P * PAGE_GROUPS, -1)
        view[m] += b
        khat[pages] = view.view(P, PAGE_GROUPS, -1)
    return khat


def make(name: str, *, B: int, ctx: int, Hq: int, Hkv: int, D: int, H_I: int, D_I: int,
         K: int, kv_dtype: str, q_dtype: str, dist: str = "normal", pages: str = "perm",
         seed: int = 0, device="cpu", q_pos=None, q_req=None, capture_pos=None,
         idx_dtype: str = "f32") -> Workload:
    """Generic generator.  Default queries: one per request at the last token
    (decode).  Pass q_pos / q_req for prefill-style query sets."""
    g = _gen(seed, device)
    ppr = (ctx + PAGE_TOKENS - 1) // PAGE_TOKENS
    page_table = page_table_for(B, ppr, pages, g, device)
    num_pages = B * ppr
    if q_pos is None:
        q_pos = torch.full((B,), ctx - 1, dtype=torch.int32, device=device)
        q_req = torch.arange(B, dtype=torch.int32, device=device)
    q_pos = torch.as_tensor(q_pos, dtype=torch.int32, device=device).contiguous()
    q_req = torch.as_tensor(q_req, dtype=torch.int32, device=device).contiguous()
    T = q_pos.numel()
    q_idx, w_idx, khat = _indexer_inputs(T, H_I, D_I, num_pages, dist, g, device, q_req, B)
    if dist == "peaked":
        khat = _add_peaks(khat, q_idx, page_table, q_req, g, device)
    if idx_dtype == "bf16":   # indexer query and keys stored as BF16 (RNE)
        q_idx, _ = _store(q_idx, "bf16")
        khat, _ = _store(khat, "bf16")
    q, _ = _store(_randn((T, Hq, D), g, device), q_dtype)
    kv_shape = (num_pages, PAGE_TOKENS, Hkv, D)
    k_pages, k_scale = _store(_randn(kv_shape, g, device), kv_dtype)
    v_pages, v_scale = _store(_randn(kv_shape, g, device), kv_dtype)
    if capture_pos is not None:
        capture_pos = torch.as_tensor(capture_pos, dtype=torch.int32, device=device).contiguous()
        extra = int((q_pos // GROUP_TOKENS - capture_pos // GROUP_TOKENS).max().item())
    else:
        extra = 0
    W = GROUP_TOKENS * K + GROUP_TOKENS + GROUP_TOKENS * max(0, extra)
    return Workload(name=name, B=B, Hq=Hq, Hkv=Hkv, D=D, H_I=H_I, D_I=D_I, K=K, W=W,
                    kv_dtype=kv_dtype, q_dtype=q_dtype, q=q, q_idx=q_idx, w_idx=w_idx,
                    k_idx_pages=khat, k_pages=k_pages, v_pages=v_pages, k_scale=k_scale,
                    v_scale=v_scale, page_table=page_table, q_req=q_req, q_pos=q_pos,
                    capture_pos=capture_pos, dist=dist, seed=seed)


def indexer_weights(hidden: int, H_I: int = 4, D_I: int = 128, seed: int = 0, device="cpu",
                    dtype: str = "bf16"):
    """Synthetic, seeded weights of the indexer's projection and of the C4
    compression (there is no checkpoint): w [H_I*D_I + H_I + D_I, hidden]
    stacking W_q, W_w, W_k with N(0, 1/hidden) entries (so projected values
    are about N(0, 1)), wphi [D_I, 4*D_I] = mean pooling [I/4 x 4] plus
    N(0, 0.02^2) entries, and bias [D_I] ~ N(0, 0.01^2).  Returns
    (w, wphi, bias); w in the given storage type, the others float32."""
    g = _gen(seed, device)
    N = H_I * D_I + H_I + D_I
    w = _randn((N, hidden), g, device) / float(hidden) ** 0.5
    eye = torch.eye(D_I, device=device, dtype=torch.float32)
    wphi = torch.cat([eye / GROUP_TOKENS] * GROUP_TOKENS, dim=1) + 0.02 * _randn((D_I, GROUP_TOKENS * D_I), g, device)
    bias = 0.01 * _randn((D_I,), g, device)
    w, _ = _store(w, dtype)
    return w, wphi.contiguous(), bias.contiguous()


def hidden_states(T: int, hidden: int, seed: int = 0, device="cpu", dtype: str = "bf16") -> torch.Tensor:
    """Synthetic hidden states x [T, hidden] ~ N(0, 1) in the given storage type."""
    x, _ = _store(_randn((T, hidden), _gen(seed, device), device), dtype)
    return x


# ---- the named workloads --------------------------------------------------------

def tiny(device="cpu", seed=0, **kw) -> Workload:
    """1 request, context 1,024 (256 groups), budget 32 groups, 4 q / 1 kv
    heads of dim 64, indexer 2 heads of dim 32, all float32, identity pages."""
    args = dict(B=1, ctx=1024, Hq=4, Hkv=1, D=64, H_I=2, D_I=32, K=32, kv_dtype="f32",
                q_dtype="f32", dist="normal", pages="identity", seed=seed, device=device)
    args.update(kw)
    return make("tiny_decode_1k", **args)


def b1_16k(device="cpu", seed=0, **kw) -> Workload:
    """B1 decode at 16,384 context, 16/2 heads of dim 256, BF16 KV, indexer
    4 heads of dim 128 (4,096 groups), budget 512 groups, permuted pages."""
    args = dict(B=1, ctx=16384, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512, kv_dtype="bf16",
                q_dtype="bf16", dist="normal", pages="perm", seed=seed, device=device)
    args.update(kw)
    return make("b1_decode_16k_bf16", **args)


def b8_262k(K=512, device="cpu", seed=0, **kw) -> Workload:
    """B8 decode at 262,144 context per request (65,536 groups), FP8 E4M3 KV
    with per-tensor scales, 16/2 heads of dim 256, peaked indexer scores."""
    args = dict(B=8, ctx=262144, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=K, kv_dtype="fp8",
                q_dtype="bf16", dist="peaked", pages="perm", seed=seed, device=device)
    args.update(kw)
    name = "262k" if args["ctx"] == 262144 else f"{args['ctx']}"
    return make(f"b8_decode_{name}_fp8_k{args['K']}", **args)


def prefill_chunk(device="cpu", seed=0, new=8192, prefix=57344, **kw) -> Workload:
    """8,192 new query tokens after a 57,344-token cached prefix (65,536 total),
    causal, 24/2 heads of dim 256, BF16, budget 512 groups (2,048 tokens); the
    indexer query and keys are BF16 (the prefill scoring pass is a BF16 GEMM)."""
    ctx = prefix + new
    q_pos = torch.arange(prefix, ctx, dtype=torch.int32)
    q_req = torch.zeros(new, dtype=torch.int32)
    args = dict(B=1, ctx=ctx, Hq=24, Hkv=2, D=256, H_I=4, D_I=128, K=512, kv_dtype="bf16",
                q_dtype="bf16", dist="normal", pages="perm", seed=seed, device=device,
                q_pos=q_pos, q_req=q_req, idx_dtype="bf16")
    args.update(kw)
    return make(f"prefill_{new}q_{ctx}ctx_bf16", **args)


def mtp(device="cpu", seed=0, ctx=4096, **kw) -> Workload:
    """MTP-style reuse: one selection captured at p0 (the last token of a
    block), two draft positions p0+1, p0+2 that fall in the next block, so the
    group completed since the capture is appended."""
    p0 = ((ctx - 6) // GROUP_TOKENS) * GROUP_TOKENS + 3   # last token of a block, p0 + 2 < ctx
    q_pos = torch.tensor([p0 + 1, p0 + 2], dtype=torch.int32)
    cap = torch.tensor([p0, p0], dtype=torch.int32)
    q_req = torch.zeros(2, dtype=torch.int32)
    args = dict(B=1, ctx=ctx, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512, kv_dtype="bf16",
                q_dtype="bf16", dist="normal", pages="perm", seed=seed, device=device,
                q_pos=q_pos, q_req=q_req, capture_pos=cap)
    args.update(kw)
    return make(f"mtp_draft2_{ctx}", **args)


SWEEP_CONTEXTS = (4096, 16384, 65536, 131072, 262144)
SWEEP_BATCHES = (1, 2, 4, 8)
SWEEP_HEADS = ((16, 2), (12, 1), (6, 1), (3, 1))
SWEEP_BUDGETS = (512, 1024, 2048)
SWEEP_KV = ("bf16", "fp8")
SWEEP_DISTS = ("normal", "peaked", "ties")

# A covering subset of the sweep's cross product (5 x 4 x 4 x 3 x 2 x 3 =
# 1,440 cases): every value of every axis appears at least once.
# (context, batch, (Hq, Hkv), budget, KV storage, score distribution)
SWEEP_CASES = (
    (4096, 1, (16, 2), 512, "bf16", "ties"),
    (4096, 8, (3, 1), 2048, "fp8", "normal"),
    (16384, 2, (12, 1), 1024, "fp8", "peaked"),
    (16384, 4, (6, 1), 2048, "bf16", "ties"),
    (65536, 4, (16, 2), 512, "fp8", "normal"),
    (65536, 1, (3, 1), 1024, "bf16", "peaked"),
    (131072, 2, (6, 1), 512, "fp8", "ties"),
    (131072, 8, (12, 1), 2048, "bf16", "normal"),
    (262144, 1, (16, 2), 2048, "bf16", "ties"),
    (262144, 2, (12, 1), 1024, "fp8", "peaked"),
)


def sweep_case(ctx, B, heads, K, kv, dist, device="cpu", seed=0) -> Workload:
    Hq, Hkv = heads
    return make(f"sweep_c{ctx}_b{B}_h{Hq}x{Hkv}_k{K}_{kv}_{dist}", B=B, ctx=ctx, Hq=Hq,
                Hkv=Hkv, D=256, H_I=4, D_I=128, K=K, kv_dtype=kv, q_dtype="bf16", dist=dist,
                pages="perm", seed=seed, device=device)

