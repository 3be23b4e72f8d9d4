"""Every buffer the library writes is written in full, and no kernel reads
memory that no kernel wrote.  A step run over poisoned outputs and
workspaces -- NaN in every float buffer, 0xFF in every byte workspace,
random integers in every id and count buffer, a random prefix histogram --
must return bit for bit what the same step returns over clean buffers.

What the contract lets a call leave alone is not compared: score entries
from a row's candidate count c on (left as they are, or -inf).  The prefix
histogram is a hint (a wrong one only costs time), and the Top-K leaves it
zero whatever it held."""
import pytest
import torch

from indexer_top_sparse_c4_b200 import workloads as wl
from indexer_top_sparse_c4_b200.pipeline import QSADraftLoop, QSAStep

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from indexer_top_sparse_c4_b200 import build
    build.build()


def _bits(t):
    """The tensor's bit patterns, so that equal NaNs compare equal."""
    t = t.detach()
    if t.dtype == torch.float32:
        return t.view(torch.int32).cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu()
    return t.cpu()


def _poison(t, gen, lo=-(2 ** 31), hi=2 ** 31 - 1):
    if t is None:
        return
    if t.dtype in (torch.float32, torch.bfloat16):
        t.fill_(float("nan"))
    elif t.dtype == torch.uint8:
        t.fill_(0xFF)
    else:
        t.copy_(torch.randint(lo, hi, t.shape, generator=gen, dtype=torch.int64).to(t.dtype))


def _step_outputs(step):
    rows = []
    c = (step.sel_pos // 4).clamp(max=step.score_stride).cpu()
    scores = _bits(step.scores)
    for t in range(step.w.T):
        rows.append(scores[t, :int(c[t])])
    return {"scores": rows, "sel": _bits(step.sel), "n_sel": _bits(step.n_sel), "tok": _bits(step.tok),
            "n_tok": _bits(step.n_tok), "out": _bits(step.out), "lse": _bits(step.lse)}


def _poison_step(step, gen):
    for t in (step.scores, step.sel, step.n_sel, step.tok, step.n_tok, step.out, step.lse, step.ws,
              step.topk_ws):
        _poison(t, gen)
    _poison(step.prefix_hist, gen, 0, 1000)   # small counts: a wrong histogram, not an overflowing one


def _same(a, b):
    assert a.keys() == b.keys()
    for k in a:
        if k == "scores":
            assert len(a[k]) == len(b[k])
            for t, (x, y) in enumerate(zip(a[k], b[k])):
                assert torch.equal(x, y), ("scores", t)
        else:
            assert torch.equal(a[k], b[k]), k


CASES = {
    "tiny_decode": lambda: wl.tiny(device="cuda"),
    "b1_decode_16k_bf16": lambda: wl.b1_16k(device="cuda"),
    "b8_decode_262k_fp8_k512": lambda: wl.b8_262k(K=512, device="cuda"),
    "b8_decode_262k_fp8_k2048": lambda: wl.b8_262k(K=2048, device="cuda"),
    "mtp_capture_reuse": lambda: wl.mtp(device="cuda"),
    "prefill_1024q_16384ctx": lambda: wl.prefill_chunk(device="cuda", new=1024, prefix=15360),
}


@pytest.mark.parametrize("case", list(CASES))
def test_step_over_poisoned_buffers(case):
    step = QSAStep(CASES[case]())
    step.run()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    clean = _step_outputs(step)
    _poison_step(step, torch.Generator().manual_seed(7))
    step.run()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    _same(clean, _step_outputs(step))
    if step.prefix_hist is not None:
        assert int(step.prefix_hist.count_nonzero().item()) == 0


@pytest.mark.parametrize("fused", [True, False])
def test_draft_loop_over_poisoned_buffers(fused):
    """The MTP draft steps, fused (stages 3 and 4 in one call, its own
    workspace) and unfused."""
    ctx, B = 262144, 8
    p0 = ((ctx - 6) // 4) * 4 + 3   # the last token of a block; the drafts p0 + 1, p0 + 2 are in the cache
    w = wl.b8_262k(K=512, device="cuda", q_pos=torch.full((B,), p0, dtype=torch.int32),
                   q_req=torch.arange(B, dtype=torch.int32))
    loop = QSADraftLoop(w, fused=fused)
    loop.run()
    torch.cuda.synchronize()
    assert int(loop.status.item()) == 0
    clean = [(_bits(o), _bits(l)) for o, l in zip(loop.out, loop.lse)]
    gen = torch.Generator().manual_seed(11)
    _poison_step(loop.capture, gen)
    for t in (*loop.out, *loop.lse, *loop.tok, *loop.n_tok, loop.ws):
        _poison(t, gen)
    loop.run()
    torch.cuda.synchronize()
    assert int(loop.status.item()) == 0
    for i, (o, l) in enumerate(zip(loop.out, loop.lse)):
        assert torch.equal(clean[i][0], _bits(o)), ("out", i)
        assert torch.equal(clean[i][1], _bits(l)), ("lse", i)
