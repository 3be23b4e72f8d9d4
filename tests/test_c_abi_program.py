"""A C program drives one decode step through libqsa.so's C ABI alone
(tests/c_abi_decode.c): the header compiles as C and links against the
library (CPU), and on a GPU the program's outputs equal the same step run
through the Python binding bit for bit, and the oracle's within the stated
tolerances."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi_decode.c")
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(out_dir):
    from indexer_top_sparse_c4_b200 import build
    lib = build.build()
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = os.path.join(out_dir, "c_abi_decode")
    libdir = os.path.dirname(lib)
    cmd = [cc, "-std=c11", "-O2", "-Wall", "-Wextra", "-Werror", SRC, "-o", exe,
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA_HOME, "include"),
           "-L", libdir, "-lqsa", "-L", os.path.join(CUDA_HOME, "lib64"), "-lcudart",
           f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{os.path.join(CUDA_HOME, 'lib64')}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    return exe


def test_c_program_builds_against_the_header_and_library(tmp_path):
    assert os.access(_compile(str(tmp_path)), os.X_OK)


@pytest.mark.gpu
def test_c_program_decode_step_matches_binding_and_oracle(tmp_path, oracle):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from indexer_top_sparse_c4_b200 import qsa
    from indexer_top_sparse_c4_b200 import workloads as wl
    from indexer_top_sparse_c4_b200.pipeline import QSAStep
    from parity_utils import (ATTN_MAX_ABS, ATTN_MEAN_ABS, ATTN_REL_L2, attn_errors, compact_pages, host,
                              out_as_f64)
    exe = _compile(str(tmp_path))
    w = wl.make("c_abi", B=2, ctx=16384, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512, kv_dtype="fp8",
                q_dtype="bf16", dist="peaked", seed=5, device="cuda")
    st = QSAStep(w)
    st.run()
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0
    ind, outd = tmp_path / "in", tmp_path / "out"
    ind.mkdir()
    outd.mkdir()
    arrays = {"q_idx": w.q_idx, "w_idx": w.w_idx, "k_idx": w.k_idx_pages, "page_table": w.page_table,
              "q_req": w.q_req, "q_pos": w.q_pos, "q": w.q, "k_pages": w.k_pages, "v_pages": w.v_pages}
    for name, t in arrays.items():
        t.contiguous().cpu().view(torch.uint8).numpy().tofile(str(ind / name))
    dims = [w.T, w.H_I, w.D_I, w.k_pages.shape[0], w.page_table.shape[0], w.page_table.shape[1], w.Hq, w.Hkv,
            w.D, w.K, w.W, st.score_stride, qsa.QSA_BF16, qsa.QSA_FP8_E4M3, qsa.QSA_BF16]
    (ind / "dims.txt").write_text(" ".join(str(int(v)) for v in dims) + f" {w.k_scale!r} {w.v_scale!r}\n")
    r = subprocess.run([exe, str(ind), str(outd)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith(f"ok abi={qsa.qsa_abi_version()}")

    def load(name, dtype, shape):
        return np.fromfile(str(outd / name), dtype=dtype).reshape(shape)

    T = w.T
    c_scores = load("scores", np.float32, (T, st.score_stride))
    c_sel, c_nsel = load("sel", np.int32, (T, w.K)), load("n_sel", np.int32, (T,))
    c_tok, c_ntok = load("tok", np.int32, (T, w.W)), load("n_tok", np.int32, (T,))
    c_out = load("out", np.uint16, (T, w.Hq, w.D))
    c_lse = load("lse", np.float32, (T, w.Hq))
    # the same kernels on the same inputs: the binding's step, bit for bit
    g_scores = host(st.scores)
    for t, c in enumerate(host(w.q_pos) // 4):   # candidates of row t (the rest of the row is not written)
        assert np.array_equal(c_scores[t, :c].view(np.uint32), g_scores[t, :c].view(np.uint32))
    assert np.array_equal(c_sel, host(st.sel)) and np.array_equal(c_nsel, host(st.n_sel))
    assert np.array_equal(c_tok, host(st.tok)) and np.array_equal(c_ntok, host(st.n_tok))
    assert np.array_equal(c_out, st.out.cpu().view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(c_lse.view(np.uint32), host(st.lse).view(np.uint32))
    # and the oracle: Top-K and expansion bit-exact on these scores, attention within tolerance
    q_pos = host(w.q_pos)
    sel_ref, nsel_ref = oracle.topk_groups(c_scores, q_pos, w.K)
    assert np.array_equal(c_sel, sel_ref) and np.array_equal(c_nsel, nsel_ref)
    tok_ref, ntok_ref, bad = oracle.expand_select(c_sel, c_nsel, q_pos, w.W, None)
    assert bad == 0 and np.array_equal(c_tok, tok_ref) and np.array_equal(c_ntok, ntok_ref)
    req = host(w.q_req)
    kc, vc, pt = compact_pages(w.k_pages, w.v_pages, w.page_table, c_tok, c_ntok, req)
    out_ref, _, sk = oracle.sparse_attn(host(w.q), kc, vc, pt, c_tok, c_ntok, w.k_scale, w.v_scale, q_req=req)
    assert sk == 0
    c_out_f = torch.from_numpy(c_out.view(np.int16)).view(torch.bfloat16)
    mx, mean, rel = attn_errors(out_as_f64(c_out_f), out_ref)
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel <= ATTN_REL_L2, (mx, mean, rel)
