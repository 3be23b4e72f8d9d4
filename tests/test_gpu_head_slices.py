"""Tensor parallelism over heads needs nothing from the library: a rank that
holds KV heads [a, b) and their query heads calls the same decode attention
on its slices, with the selection every rank computes alike (the indexer is
replicated).  The two halves of a B8 decode step, each through its own call,
must give the full call's output and LSE on their heads: the same tokens and
the same math, only the split of each row over CTAs differs.  The softmax
weights enter the PV product in f16, relative to each chunk's running
maximum, so with other chunk boundaries each weight rounds differently (2^-11
relative): the outputs differ by about 2^-11 of the V scale plus the BF16
rounding of the output -- bounded here at 2e-3 (max) and 2e-4 (mean), ten
times below the attention tolerance against the oracle; the LSE sums run in
FP32 and agree to 1e-5."""
import numpy as np
import pytest
import torch

from indexer_top_sparse_c4_b200 import workloads as wl
from indexer_top_sparse_c4_b200.pipeline import QSAStep
from parity_utils import host, out_as_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from indexer_top_sparse_c4_b200 import build, qsa
    build.build()
    return qsa


@pytest.mark.parametrize("kv, K", [("fp8", 512), ("bf16", 2048)])
def test_head_slices_reproduce_the_full_call(q, kv, K):
    w = wl.make("heads", B=8, ctx=16384, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=K, kv_dtype=kv, q_dtype="bf16",
                dist="peaked", seed=31, device="cuda")
    st = QSAStep(w)
    st.run()
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0
    full, full_lse = out_as_f64(st.out), host(st.lse)
    G = w.Hq // w.Hkv
    for r in range(w.Hkv):                      # one "rank" per KV head
        heads = slice(r * G, (r + 1) * G)
        qs = w.q[:, heads].contiguous()
        ks = w.k_pages[:, :, r:r + 1].contiguous()
        vs = w.v_pages[:, :, r:r + 1].contiguous()
        out = torch.empty((w.T, G, w.D), dtype=st.out.dtype, device="cuda")
        lse = torch.empty((w.T, G), dtype=torch.float32, device="cuda")
        ws_bytes = q.qsa_sparse_attn_decode_workspace_size(w.T, G, 1, w.D, w.W, ks.dtype)
        ws = torch.empty((max(ws_bytes, 16),), dtype=torch.uint8, device="cuda")
        status = torch.zeros((1,), dtype=torch.int32, device="cuda")
        q.qsa_sparse_attn_decode(qs, ks, vs, w.page_table, st.tok, st.n_tok, out, workspace=ws,
                                 k_scale=w.k_scale, v_scale=w.v_scale, q_req=w.q_req, lse=lse, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got = out_as_f64(out)
        ref = full[:, heads]
        diff = np.abs(got - ref)
        assert diff.max() <= 2e-3 and diff.mean() <= 2e-4, (float(diff.max()), float(diff.mean()))
        np.testing.assert_allclose(host(lse), full_lse[:, heads], rtol=1e-5, atol=1e-5)
