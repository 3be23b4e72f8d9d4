"""One QSA step over a Workload: device buffers (allocated once with torch) and
the four library calls in order on one stream.

    scores  <- qsa_index_scores      (query position, or the capture position
                                       when an MTP draft reuses a selection)
    sel     <- qsa_topk_groups
    tok     <- qsa_expand_select
    out     <- qsa_sparse_attn_decode / qsa_sparse_attn_prefill

This is plumbing only: torch provides memory and the stream, libqsa.so does
all the work.
"""
from __future__ import annotations

import torch

from . import qsa
from .workloads import GROUP_TOKENS, Workload


class QSAStep:
    """seq_len_threshold (TensorRT-LLM "QSASparseAttentionConfig"): queries
    whose sequence has at most this many tokens attend densely to all of
    them; None or a value below the token budget 4*K means the budget, which
    the Top-K's dense fallback (c <= K) already honours, so no extra launch is
    made then."""

    def __init__(self, w: Workload, prefill: bool | None = None, out_dtype=None,
                 score_stride: int | None = None, prefix_hist: bool | None = None,
                 seq_len_threshold: int | None = None):
        self.w = w
        dev = w.q.device
        self.threshold = qsa.qsa_seq_len_threshold(seq_len_threshold, w.K)
        # an explicit threshold above the budget: dense rows up to that many tokens
        self.dense_rows = self.threshold > GROUP_TOKENS * w.K
        if self.dense_rows and self.threshold > w.W:
            w.W = self.threshold
        self.prefill = (w.T > 64) if prefill is None else prefill
        self.sel_pos = w.capture_pos if w.capture_pos is not None else w.q_pos
        if score_stride is None:
            # the largest candidate count, rounded up to 4 so that every score
            # row starts on 16 bytes
            score_stride = -(-max(1, int(self.sel_pos.max().item()) // GROUP_TOKENS) // 4) * 4
        self.score_stride = score_stride
        T = w.T
        self.scores = torch.empty((T, self.score_stride), dtype=torch.float32, device=dev)
        self.sel = torch.empty((T, w.K), dtype=torch.int32, device=dev)
        self.n_sel = torch.empty((T,), dtype=torch.int32, device=dev)
        self.tok = torch.empty((T, w.W), dtype=torch.int32, device=dev)
        self.n_tok = torch.empty((T,), dtype=torch.int32, device=dev)
        if out_dtype is None:
            out_dtype = torch.float32 if w.q.dtype == torch.float32 else torch.bfloat16
        self.out = torch.empty((T, w.Hq, w.D), dtype=out_dtype, device=dev)
        self.lse = torch.empty((T, w.Hq), dtype=torch.float32, device=dev)
        self.status = torch.zeros((1,), dtype=torch.int32, device=dev)
        ws = 0 if self.prefill else qsa.qsa_sparse_attn_decode_workspace_size(
            T, w.Hq, w.Hkv, w.D, w.W, w.k_pages.dtype)
        self.ws_bytes = ws   # > 0: split-K partials and one combine kernel per call
        self.ws = torch.empty((max(ws, 16),), dtype=torch.uint8, device=dev)
        tk = qsa.qsa_topk_groups_workspace_size(T, w.K, self.score_stride)
        self.topk_ws = torch.empty((max(tk, 16),), dtype=torch.uint8, device=dev) if tk else None
        # the scan's 12-bit key-prefix counts, handed to the Top-K (decode rows);
        # zero at allocation, and every Top-K call leaves it zero again
        if prefix_hist is None:
            prefix_hist = not self.prefill
        self.prefix_hist = (torch.zeros((T, qsa.QSA_PREFIX_HIST_BINS), dtype=torch.int32, device=dev)
                            if prefix_hist else None)

    # the four stages, separately callable for per-stage tests and timing
    def index_scores(self, stream=None):
        w = self.w
        qsa.qsa_index_scores(w.q_idx, w.w_idx, w.k_idx_pages, w.page_table, self.sel_pos,
                             self.scores, q_req=w.q_req, dev_status=self.status, stream=stream,
                             prefix_hist=self.prefix_hist)

    def topk(self, stream=None):
        qsa.qsa_topk_groups(self.scores, self.sel_pos, self.w.K, self.sel, self.n_sel,
                            workspace=self.topk_ws, dev_status=self.status, stream=stream,
                            prefix_hist=self.prefix_hist)

    def expand(self, stream=None):
        w = self.w
        qsa.qsa_expand_select(self.sel, self.n_sel, w.q_pos, self.tok, self.n_tok,
                              capture_pos=w.capture_pos, dev_status=self.status, stream=stream)

    def attention(self, stream=None, sm_scale=0.0):
        w = self.w
        common = dict(k_scale=w.k_scale, v_scale=w.v_scale, q_req=w.q_req, sm_scale=sm_scale,
                      lse=self.lse, dev_status=self.status, stream=stream)
        if self.prefill:
            qsa.qsa_sparse_attn_prefill(w.q, w.k_pages, w.v_pages, w.page_table, self.tok,
                                        self.n_tok, self.out, **common)
        else:
            qsa.qsa_sparse_attn_decode(w.q, w.k_pages, w.v_pages, w.page_table, self.tok,
                                       self.n_tok, self.out, workspace=self.ws, **common)

    def select(self, stream=None):
        """Top-K and expansion: one launch when there is no MTP capture; then
        the dense rows of an explicit sequence-length threshold."""
        w = self.w
        if w.capture_pos is None:
            qsa.qsa_topk_expand(self.scores, w.q_pos, w.K, self.sel, self.n_sel, self.tok, self.n_tok,
                                dev_status=self.status, stream=stream, prefix_hist=self.prefix_hist)
        else:
            self.topk(stream)
            self.expand(stream)
        if self.dense_rows:
            self.dense_select(self.threshold, stream)

    def dense_select(self, threshold, stream=None):
        qsa.qsa_dense_select(self.w.q_pos, threshold, self.tok, self.n_tok, dev_status=self.status, stream=stream)

    def run(self, stream=None, sm_scale=0.0):
        self.index_scores(stream)
        self.select(stream)
        self.attention(stream, sm_scale)
        return self.out

    def bind(self, stream=None, sm_scale=0.0):
        """run()'s library calls with their arguments converted once: a
        callable that only crosses into C (for loops where the host issues
        every step).  It names this step's tensors as they are now: bind
        again after replacing one; refilling them in place is fine."""
        if stream is None:
            stream = torch.cuda.current_stream()
        return qsa.bind(self.run, stream, sm_scale)


class QSADecodeGraphs:
    """The two decode graph families of the sequence-length threshold
    (TensorRT-LLM "QSASparseAttentionConfig",
    needs_separate_short_long_cuda_graphs): one CUDA graph of a step for
    batches whose every sequence is at most the threshold -- dense attention
    over every token, no indexer and no Top-K launched -- and one of the full
    QSA step (rows at or below the threshold still dense) for the others.
    The caller updates the step's inputs in place and replays the family
    its batch needs; the host knows the sequence lengths of its batch."""

    def __init__(self, step: QSAStep, stream=None):
        if step.prefill or step.w.capture_pos is not None:
            raise ValueError("decode steps without an MTP capture")
        self.step = step
        self.stream = stream if stream is not None else torch.cuda.Stream(step.w.q.device)
        big = 1 << 30                    # every row dense
        with torch.cuda.stream(self.stream):
            # warm-up outside the capture (first-call set-up of every kernel);
            # the dense rows of the step's own threshold always fit its lists
            step.run()
            step.dense_select(step.threshold)
            torch.cuda.synchronize()
            self.dense = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.dense, stream=self.stream):
                step.dense_select(big, self.stream)
                step.attention(self.stream)
            self.sparse = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.sparse, stream=self.stream):
                step.run(self.stream)

    def family(self, max_seq_len: int) -> str:
        return "dense" if max_seq_len <= self.step.threshold else "sparse"

    def replay(self, max_seq_len: int):
        """Replays the family of a batch whose longest sequence has
        max_seq_len tokens (on the graphs' stream); returns its name."""
        fam = self.family(max_seq_len)
        if fam == "dense" and max_seq_len > self.step.w.W:
            raise ValueError("a dense batch wider than the step's token lists")
        (self.dense if fam == "dense" else self.sparse).replay()
        return fam


class QSADraftLoop:
    """The MTP draft loop with index sharing (TensorRT-LLM
    "QSASparseAttentionConfig", the MTP index-sharing field): the capture
    step at p0 scores, selects and attends like any decode step; each of the
    `drafts` draft steps at p0 + i reuses the captured selection, with the
    groups completed since p0 appended (qsa_expand_select with capture_pos),
    and only attends.  The indexer does not run again during the loop.

    Draft step i has one row per capture row (the same request), its own
    attention query (seeded, the capture query's dtype and shape) and its own
    output.  fused (default): each draft step is one qsa_sparse_attn_decode_sel
    call (stages 3 and 4 together, no token lists); otherwise the expansion
    writes the draft's token lists and qsa_sparse_attn_decode reads them.
    Plumbing only: every stage is a libqsa call."""

    def __init__(self, w: Workload, drafts: int = 2, seed: int = 1, fused: bool = True):
        if w.capture_pos is not None:
            raise ValueError("the capture workload is a plain decode workload")
        self.w = w
        self.drafts = drafts
        self.capture = QSAStep(w)
        dev = w.q.device
        g = torch.Generator(device="cpu").manual_seed(seed)
        T = w.T
        c0 = w.q_pos // GROUP_TOKENS
        self.pos = [(w.q_pos + i).contiguous() for i in range(1, drafts + 1)]
        extra = int((self.pos[-1] // GROUP_TOKENS - c0).max().item())  # groups completed since p0
        self.W = GROUP_TOKENS * w.K + GROUP_TOKENS + GROUP_TOKENS * max(0, extra)
        self.q = [torch.randn(w.q.shape, generator=g).to(dtype=w.q.dtype, device=dev) for _ in range(drafts)]
        self.tok = [torch.empty((T, self.W), dtype=torch.int32, device=dev) for _ in range(drafts)]
        self.n_tok = [torch.empty((T,), dtype=torch.int32, device=dev) for _ in range(drafts)]
        self.out = [torch.empty_like(self.capture.out) for _ in range(drafts)]
        self.lse = [torch.empty_like(self.capture.lse) for _ in range(drafts)]
        self.fused = fused
        size = qsa.qsa_sparse_attn_decode_sel_workspace_size if fused else qsa.qsa_sparse_attn_decode_workspace_size
        ws = size(T, w.Hq, w.Hkv, w.D, self.W, w.k_pages.dtype)
        self.ws = torch.empty((max(ws, 16),), dtype=torch.uint8, device=dev)
        self.status = self.capture.status

    def draft_step(self, i: int, stream=None, sm_scale=0.0):
        w, cap = self.w, self.capture
        if self.fused:
            qsa.qsa_sparse_attn_decode_sel(self.q[i], w.k_pages, w.v_pages, w.page_table, cap.sel, cap.n_sel,
                                           self.pos[i], self.W, self.out[i], workspace=self.ws,
                                           capture_pos=w.q_pos, k_scale=w.k_scale, v_scale=w.v_scale,
                                           q_req=w.q_req, sm_scale=sm_scale, lse=self.lse[i],
                                           dev_status=self.status, stream=stream)
            return
        qsa.qsa_expand_select(cap.sel, cap.n_sel, self.pos[i], self.tok[i], self.n_tok[i],
                              capture_pos=w.q_pos, dev_status=self.status, stream=stream)
        qsa.qsa_sparse_attn_decode(self.q[i], w.k_pages, w.v_pages, w.page_table, self.tok[i],
                                   self.n_tok[i], self.out[i], workspace=self.ws, k_scale=w.k_scale,
                                   v_scale=w.v_scale, q_req=w.q_req, sm_scale=sm_scale,
                                   lse=self.lse[i], dev_status=self.status, stream=stream)

    def run(self, stream=None, sm_scale=0.0):
        self.capture.run(stream, sm_scale)
        for i in range(self.drafts):
            self.draft_step(i, stream, sm_scale)
        return [self.capture.out] + self.out
