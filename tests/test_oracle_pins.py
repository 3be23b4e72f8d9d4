"""Pins for the CPU oracle: checks against things other than the oracle itself
(hand-worked values, library routines a special case reduces to, brute force
on tiny inputs, invariants the method fixes).  CPU only."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from indexer_top_sparse_c4_b200 import workloads as wl

HERE = os.path.dirname(os.path.abspath(__file__))


# ---- value decoders -------------------------------------------------------------

def test_e4m3_all_256_codes_match_torch(oracle):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_f64(i) for i in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2                      # 0x7F and 0xFF only
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_bf16_decode_matches_torch(oracle):
    g = torch.Generator().manual_seed(1)
    bits = torch.randint(0, 65536, (4096,), generator=g, dtype=torch.int32)
    bits = bits[(bits & 0x7F80) != 0x7F80]     # skip inf/nan patterns
    ref = bits.to(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_f64(int(b)) for b in bits])
    assert np.array_equal(ref, got)


# ---- stage 1: scores ------------------------------------------------------------

def _read_golden(name):
    vals = {}
    for line in open(os.path.join(HERE, "golden", name)):
        line = line.split("#")[0].strip()
        if line:
            k, v = line.split("=")
            vals[k.strip()] = [float(x) for x in v.split()]
    return vals


def test_scores_hand_worked_example(oracle):
    gv = _read_golden("scores_worked_example.txt")
    q = np.array([[gv["q_h0"], gv["q_h1"]]], np.float32)          # [1, 2, 2]
    w = np.array([gv["w"]], np.float32)
    khat = np.zeros((2, 16, 2), np.float32)
    # the three groups live in logical page 0 -> physical page 1
    khat[1, 0], khat[1, 1], khat[1, 2] = gv["khat_g0"], gv["khat_g1"], gv["khat_g2"]
    khat[0] = 99.0                                                  # decoy page
    pt = np.array([[1]], np.int32)
    s, skipped = oracle.index_scores(q, w, khat, pt, np.array([13], np.int32), score_stride=4)
    assert skipped == 0
    assert s[0, :3].tolist() == gv["expected"]
    assert s[0, 3] == -np.inf                                       # current block not scored


def test_scores_all_positive_reduce_to_bilinear_form(oracle):
    """With every q_h . khat_g > 0 the ReLU vanishes and s = w^T Q khat, a
    plain matrix product."""
    rng = np.random.default_rng(3)
    H, D, G = 4, 128, 64
    q = np.abs(rng.standard_normal((1, H, D))).astype(np.float32)
    khat = np.abs(rng.standard_normal((4, 16, D))).astype(np.float32)
    w = rng.random((1, H)).astype(np.float32)
    pt = np.array([[2, 0, 3, 1]], np.int32)
    s, _ = oracle.index_scores(q, w, khat, pt, np.array([4 * G + 1], np.int32))
    logical = khat[pt[0]].reshape(G, D).astype(np.float64)
    ref = (w.astype(np.float64) @ (q[0].astype(np.float64) @ logical.T))[0]
    assert np.array_equal(s[0, :G], ref.astype(np.float32))


def test_scores_relu_drops_negative_heads(oracle):
    """Negating a head whose dots are all negative leaves the scores unchanged
    only if that head contributed nothing -- i.e. the ReLU is applied per head
    before the weighted sum."""
    rng = np.random.default_rng(4)
    D = 32
    khat = np.abs(rng.standard_normal((1, 16, D))).astype(np.float32)
    q = np.abs(rng.standard_normal((1, 2, D))).astype(np.float32)
    q[0, 1] *= -1                                  # head 1: every dot < 0
    w = np.array([[0.75, 0.5]], np.float32)
    pt = np.array([[0]], np.int32)
    pos = np.array([63], np.int32)
    s, _ = oracle.index_scores(q, w, khat, pt, pos)
    q1 = q.copy()
    q1[0, 1] = 0
    s1, _ = oracle.index_scores(q1, w, khat, pt, pos)
    assert np.array_equal(s, s1)
    ref = 0.75 * (khat[0].astype(np.float64) @ q[0, 0].astype(np.float64))
    assert np.array_equal(s[0, :15], ref[:15].astype(np.float32))


def test_scores_page_table_invariance(oracle):
    """The same logical keys stored under two different page tables score the same."""
    w8 = wl.make("t", B=2, ctx=1000, Hq=2, Hkv=1, D=64, H_I=2, D_I=32, K=8, kv_dtype="f32",
                 q_dtype="f32", pages="perm", seed=5)
    n = w8.numpy()
    s_perm, _ = oracle.index_scores(n["q_idx"], n["w_idx"], n["k_idx_pages"], n["page_table"],
                                    n["q_pos"], n["q_req"])
    # rebuild an identity-paged copy of the same logical data
    pt = n["page_table"]
    khat_id = n["k_idx_pages"][pt.reshape(-1)]
    pt_id = np.arange(pt.size, dtype=np.int32).reshape(pt.shape)
    s_id, _ = oracle.index_scores(n["q_idx"], n["w_idx"], khat_id, pt_id, n["q_pos"], n["q_req"])
    assert np.array_equal(s_perm, s_id)


def test_scores_dyadic_inputs_are_exact(oracle):
    """On the dyadic grid every partial sum is an exact float; compare with
    exact rational arithmetic done independently in Python."""
    from fractions import Fraction
    w8 = wl.make("t", B=1, ctx=256, Hq=2, Hkv=1, D=64, H_I=4, D_I=128, K=8, kv_dtype="f32",
                 q_dtype="f32", dist="dyadic", pages="perm", seed=6)
    n = w8.numpy()
    s, _ = oracle.index_scores(n["q_idx"], n["w_idx"], n["k_idx_pages"], n["page_table"], n["q_pos"])
    c = 255 // 4
    for g in range(c):
        page = n["page_table"][0, g // 16]
        k = n["k_idx_pages"][page, g % 16]
        tot = Fraction(0)
        for h in range(4):
            d = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(n["q_idx"][0, h], k))
            tot += Fraction(float(n["w_idx"][0, h])) * max(d, Fraction(0))
        assert Fraction(float(s[0, g])) == tot


def test_scores_out_of_range_page_is_skipped(oracle):
    q = np.ones((1, 1, 4), np.float32)
    w = np.ones((1, 1), np.float32)
    khat = np.ones((1, 16, 4), np.float32)
    pt = np.array([[0, 7]], np.int32)               # logical page 1 -> bad id 7
    s, skipped = oracle.index_scores(q, w, khat, pt, np.array([128], np.int32))
    assert skipped == 16
    assert np.all(s[0, :16] == 4.0) and np.all(s[0, 16:] == -np.inf)


# ---- stage 2: Top-K -------------------------------------------------------------

def _dominates(s, S, n):
    """Exactly one subset S of size min(K,n) has every member ranked above
    every non-member under (score desc, id asc)."""
    inside = set(S)
    for i in inside:
        for j in range(n):
            if j in inside:
                continue
            if not (s[i] > s[j] or (s[i] == s[j] and i < j)):
                return False
    return True


@pytest.mark.parametrize("seed", range(12))
def test_topk_brute_force_tiny(oracle, seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 11))
    K = int(rng.integers(1, 6))
    s = rng.integers(0, 4, n).astype(np.float32)        # heavy ties
    if seed % 3 == 0:
        s = rng.standard_normal(n).astype(np.float32)
    row = np.full((1, 12), -np.inf, np.float32)
    row[0, :n] = s
    pos = np.array([4 * n + int(rng.integers(0, 4))], np.int32)
    sel, n_sel = oracle.topk_groups(row, pos, K)
    m = min(K, n)
    winners = [S for S in itertools.combinations(range(n), m) if _dominates(s, S, n)]
    assert len(winners) == 1
    assert n_sel[0] == m
    assert sel[0, :m].tolist() == list(winners[0])
    assert np.all(sel[0, m:] == -1)


def test_topk_matches_library_sort(oracle):
    rng = np.random.default_rng(7)
    T, G, K = 6, 3000, 257
    s = (rng.integers(0, 64, (T, G)) / 8).astype(np.float32)   # many ties
    pos = np.array([4 * G - 1, 4 * G, 401, 4 * 1000 + 2, 4 * G - 4, 4 * 257], np.int32)
    pos = np.minimum(pos, 4 * G + 3)
    sel, n_sel = oracle.topk_groups(s, pos, K)
    for t in range(T):
        c = min(pos[t] // 4, G)
        order = np.lexsort((np.arange(c), -s[t, :c].astype(np.float64)))
        ref = np.sort(order[:min(K, c)])
        assert n_sel[t] == len(ref)
        assert np.array_equal(sel[t, :n_sel[t]], ref)


def test_topk_negative_zero_ties_with_positive_zero(oracle):
    s = np.array([[-0.0, 0.0, -1.0]], np.float32)
    sel, _ = oracle.topk_groups(s, np.array([12], np.int32), 1)
    assert sel[0, 0] == 0                      # -0 == +0, lower index wins


def test_topk_dense_fallback_when_budget_covers_all(oracle):
    s = np.random.default_rng(8).standard_normal((1, 40)).astype(np.float32)
    sel, n_sel = oracle.topk_groups(s, np.array([4 * 40 + 1], np.int32), 64)
    assert n_sel[0] == 40 and sel[0, :40].tolist() == list(range(40)) and np.all(sel[0, 40:] == -1)


# ---- stage 3: expand ------------------------------------------------------------

@pytest.mark.parametrize("p", [0, 1, 2, 3, 4, 63, 64, 1021, 1022, 1023, 1024])
def test_expand_invariants(oracle, p):
    K = 8
    c = p // 4
    rng = np.random.default_rng(p)
    n = min(K, c)
    sel = np.full((1, K), -1, np.int32)
    sel[0, :n] = np.sort(rng.choice(c, n, replace=False)) if c else []
    tok, n_tok, bad = oracle.expand_select(sel, np.array([n], np.int32), np.array([p], np.int32), 4 * K + 4)
    assert bad == 0
    row = tok[0, :n_tok[0]]
    assert n_tok[0] == 4 * n + (p - 4 * c + 1)
    assert p in row and np.all(np.diff(row) > 0)               # ascending, no duplicates
    assert set(range(4 * c, p + 1)) <= set(row.tolist())        # current block always present
    assert row.max() == p                                       # nothing from the future
    assert np.all(tok[0, n_tok[0]:] == -1)


def test_expand_mtp_appends_completed_groups(oracle):
    # captured at p0 = 4091 (c0 = 1022); drafts at 4092, 4093 (c = 1023)
    K = 4
    sel = np.array([[5, 9, 100, 1021]] * 2, np.int32)
    tok, n_tok, bad = oracle.expand_select(sel, np.array([4, 4], np.int32),
                                           np.array([4092, 4093], np.int32), 4 * K + 8,
                                           capture_pos=np.array([4091, 4091], np.int32))
    assert bad == 0
    assert tok[0, 16:20].tolist() == [4088, 4089, 4090, 4091]    # group 1022 appended
    assert tok[0, 20] == 4092 and n_tok[0] == 21
    assert tok[1, 20:22].tolist() == [4092, 4093] and n_tok[1] == 22


def test_expand_invalid_group_becomes_padding(oracle):
    sel = np.array([[3, 50]], np.int32)              # 50 >= c = 10
    tok, n_tok, bad = oracle.expand_select(sel, np.array([2], np.int32), np.array([41], np.int32), 12)
    assert bad == 1
    assert tok[0, :4].tolist() == [12, 13, 14, 15] and tok[0, 4:8].tolist() == [-1] * 4
    assert tok[0, 8:10].tolist() == [40, 41] and n_tok[0] == 10


# ---- stage 4: attention ---------------------------------------------------------

def _dense_sdpa(n, t, Hkv, upto):
    """Causal attention of query t over tokens 0..upto with torch SDPA in fp64."""
    pt = n["page_table"][n["q_req"][t] if n["q_req"] is not None else t]
    def dec(x):
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).double()
        return torch.from_numpy(x).double()
    K = dec(n["k_pages"])[pt].reshape(-1, Hkv, n["k_pages"].shape[-1])[: upto + 1]
    V = dec(n["v_pages"])[pt].reshape(-1, Hkv, n["v_pages"].shape[-1])[: upto + 1]
    q = dec(n["q"])[t]                                           # [Hq, D]
    o = torch.nn.functional.scaled_dot_product_attention(
        q[:, None, :], K.transpose(0, 1), V.transpose(0, 1), enable_gqa=True)
    return o[:, 0, :].numpy()


@pytest.mark.parametrize("kv", ["f32", "bf16"])
def test_attention_budget_covering_all_groups_is_dense_causal(oracle, kv):
    """Budget >= every complete group: QSA selects every visible token, so it
    equals plain causal attention (torch SDPA, fp64)."""
    w = wl.make("t", B=2, ctx=300, Hq=4, Hkv=2, D=64, H_I=2, D_I=32, K=80, kv_dtype=kv,
                q_dtype=kv, pages="perm", seed=9, q_pos=[299, 257], q_req=[0, 1])
    n = w.numpy()
    r = oracle.qsa_step(n["q"], n["q_idx"], n["w_idx"], n["k_idx_pages"], n["k_pages"],
                        n["v_pages"], n["page_table"], n["q_pos"], w.K, q_req=n["q_req"])
    for t in range(2):
        ref = _dense_sdpa(n, t, 2, int(n["q_pos"][t]))
        assert np.abs(r["out"][t] - ref).max() < 1e-12


def test_attention_layout_identity(oracle):
    """softmax(s*[Q,0][K,V]^T)[K,V] = [P K, P V] with the D=256 scale kept
    (the [K,V]/[Q,0] packing of the Ascend CANN prefill adapter)."""
    w = wl.make("t", B=1, ctx=200, Hq=2, Hkv=1, D=256, H_I=2, D_I=32, K=8, kv_dtype="f32",
                q_dtype="f32", pages="perm", seed=10)
    n = w.numpy()
    T = 1
    tok = np.array([[0, 5, 17, 64, 65, 130, 199, -1]], np.int32)
    n_tok = np.array([7], np.int32)
    out, lse, _ = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], tok, n_tok)
    q2 = np.concatenate([n["q"], np.zeros_like(n["q"])], axis=-1)
    kv = np.concatenate([n["k_pages"], n["v_pages"]], axis=-1)
    out2, lse2, _ = oracle.sparse_attn(q2, kv, kv, n["page_table"], tok, n_tok, sm_scale=1 / 16.0)
    assert np.abs(out2[..., 256:] - out).max() < 1e-12
    assert np.abs(lse2 - lse).max() < 1e-12
    # the K half is P.K: recompute P from the lse and check against it
    pk, _, _ = oracle.sparse_attn(n["q"], n["k_pages"], n["k_pages"], n["page_table"], tok, n_tok)
    assert np.abs(out2[..., :256] - pk).max() < 1e-12
    assert T == 1


def test_attention_order_and_paging_invariance(oracle):
    w = wl.make("t", B=1, ctx=500, Hq=6, Hkv=1, D=64, H_I=2, D_I=32, K=8, kv_dtype="bf16",
                q_dtype="bf16", pages="perm", seed=11)
    n = w.numpy()
    rng = np.random.default_rng(11)
    toks = np.sort(rng.choice(500, 37, replace=False)).astype(np.int32)
    tok = np.concatenate([toks, [-1, -1, -1]])[None].astype(np.int32)
    a, la, _ = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], tok, np.array([40]))
    shuf = tok.copy()
    rng.shuffle(shuf[0])
    b, lb, _ = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], shuf, np.array([40]))
    assert np.abs(a - b).max() < 1e-12 and np.abs(la - lb).max() < 1e-12
    pt = n["page_table"]
    pid = np.arange(pt.size, dtype=np.int32).reshape(pt.shape)
    c, lc, _ = oracle.sparse_attn(n["q"], n["k_pages"][pt[0]], n["v_pages"][pt[0]], pid, tok, np.array([40]))
    assert np.array_equal(a, c) and np.array_equal(la, lc)


def test_attention_single_token_returns_v_and_lse(oracle):
    w = wl.make("t", B=1, ctx=128, Hq=4, Hkv=2, D=64, H_I=2, D_I=32, K=8, kv_dtype="fp8",
                q_dtype="bf16", pages="perm", seed=12)
    n = w.numpy()
    tok = np.array([[77, -1]], np.int32)
    out, lse, _ = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], tok,
                                     np.array([2]), w.k_scale, w.v_scale)
    page = n["page_table"][0, 1]
    codes = torch.from_numpy(n["v_pages"][page, 77 % 64]).view(torch.float8_e4m3fn).double().numpy()
    v = codes * w.v_scale                                          # [Hkv, D]
    for h in range(4):
        assert np.array_equal(out[0, h], v[h // 2])
    kc = torch.from_numpy(n["k_pages"][page, 77 % 64]).view(torch.float8_e4m3fn).double().numpy()
    qd = torch.from_numpy(n["q"].view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    for h in range(4):
        ref = (qd[0, h] @ (kc[h // 2] * w.k_scale)) / 8.0
        assert abs(lse[0, h] - ref) < 1e-12


def test_attention_empty_rows_are_zero(oracle):
    w = wl.make("t", B=1, ctx=64, Hq=2, Hkv=1, D=64, H_I=2, D_I=32, K=8, kv_dtype="f32",
                q_dtype="f32", seed=13)
    n = w.numpy()
    for tok, nt in [(np.array([[5, 6]], np.int32), 0), (np.array([[-1, -1]], np.int32), 2)]:
        out, lse, _ = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], tok,
                                         np.array([nt]))
        assert np.all(out == 0) and np.all(lse == -np.inf)


def test_attention_lse_matches_logsumexp(oracle):
    w = wl.make("t", B=1, ctx=256, Hq=2, Hkv=1, D=64, H_I=2, D_I=32, K=8, kv_dtype="f32",
                q_dtype="f32", pages="identity", seed=14)
    n = w.numpy()
    tok = np.arange(0, 256, 3, dtype=np.int32)[None]
    out, lse, _ = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], tok,
                                     np.array([tok.shape[1]]), sm_scale=0.3)
    K = torch.from_numpy(n["k_pages"]).double().reshape(-1, 64)[tok[0]]
    V = torch.from_numpy(n["v_pages"]).double().reshape(-1, 64)[tok[0]]
    q = torch.from_numpy(n["q"][0]).double()
    logits = float(np.float32(0.3)) * q @ K.T          # the scale crosses the ABI as a float
    assert np.abs(lse[0] - torch.logsumexp(logits, -1).numpy()).max() < 1e-12
    assert np.abs(out[0] - (torch.softmax(logits, -1) @ V).numpy()).max() < 1e-12


def test_attention_fp8_scale_is_linear(oracle):
    w = wl.make("t", B=1, ctx=128, Hq=2, Hkv=1, D=64, H_I=2, D_I=32, K=8, kv_dtype="fp8",
                q_dtype="bf16", seed=15)
    n = w.numpy()
    tok = np.arange(0, 128, 5, dtype=np.int32)[None]
    nt = np.array([tok.shape[1]])
    a, _, _ = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], tok, nt, 0.5, 0.25)
    b, _, _ = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], tok, nt, 0.5, 0.5)
    assert np.abs(2 * a - b).max() < 1e-12


def test_attention_invalid_tokens_are_skipped(oracle):
    w = wl.make("t", B=1, ctx=128, Hq=2, Hkv=1, D=64, H_I=2, D_I=32, K=8, kv_dtype="f32",
                q_dtype="f32", seed=16)
    n = w.numpy()
    good = np.array([[3, 70]], np.int32)
    bad = np.array([[3, -5, 70, 128 * 7]], np.int32)
    a, _, s0 = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], good, np.array([2]))
    b, _, s1 = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], bad, np.array([4]))
    assert s0 == 0 and s1 == 2 and np.array_equal(a, b)


# ---- whole chain ----------------------------------------------------------------

def test_chain_tiny_config_runs_and_selects_budget(oracle):
    w = wl.tiny()
    n = w.numpy()
    r = oracle.qsa_step(n["q"], n["q_idx"], n["w_idx"], n["k_idx_pages"], n["k_pages"],
                        n["v_pages"], n["page_table"], n["q_pos"], w.K)
    assert r["n_sel"][0] == 32 and r["n_tok"][0] == 4 * 32 + 4
    assert r["tok"][0, r["n_tok"][0] - 1] == 1023
    assert np.isfinite(r["out"]).all()
    # the kept groups are the 32 best scores
    s = r["scores"][0, :255]
    kept = set(r["sel"][0, :32].tolist())
    thr = min(s[list(kept)])
    assert all(s[g] <= thr for g in range(255) if g not in kept)


def test_chain_mtp_reuse(oracle):
    w = wl.mtp(ctx=512)
    n = w.numpy()
    r = oracle.qsa_step(n["q"], n["q_idx"], n["w_idx"], n["k_idx_pages"], n["k_pages"],
                        n["v_pages"], n["page_table"], n["q_pos"], 64, q_req=n["q_req"],
                        capture_pos=n["capture_pos"])
    p0 = int(n["capture_pos"][0])
    assert p0 % 4 == 3
    for t in range(2):
        row = r["tok"][t, :r["n_tok"][t]]
        assert list(range(p0 - 3, p0 + 1)) == [x for x in row if p0 - 3 <= x <= p0]
        assert row[-1] == n["q_pos"][t]


def test_sm_scale_default_is_inverse_sqrt_d(oracle):
    w = wl.make("t", B=1, ctx=64, Hq=1, Hkv=1, D=64, H_I=2, D_I=32, K=8, kv_dtype="f32",
                q_dtype="f32", seed=17)
    n = w.numpy()
    tok = np.array([[1, 2, 3]], np.int32)
    a, _, _ = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], tok, np.array([3]))
    b, _, _ = oracle.sparse_attn(n["q"], n["k_pages"], n["v_pages"], n["page_table"], tok, np.array([3]),
                                 sm_scale=1 / math.sqrt(64))
    assert np.array_equal(a, b)


# ---- before stage 1: indexer projection and the C4 compressed-key write ----------

def _bf16_bits(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_projection_hand_worked(oracle):
    """y = x . w^T worked by hand: x = [[1, 2], [3, 4]], w rows (1, 0),
    (0.5, -1), (2, 2) give [[1, -1.5, 6], [3, -2.5, 14]] (every value exact in
    BF16 and FP32)."""
    x = np.array([[1, 2], [3, 4]], np.float32)
    w = np.array([[1, 0], [0.5, -1], [2, 2]], np.float32)
    want = np.array([[1, -1.5, 6], [3, -2.5, 14]], np.float32)
    assert np.array_equal(oracle.indexer_project(x, w), want)
    assert np.array_equal(oracle.indexer_project(_bf16_bits(x), _bf16_bits(w)), want)


def test_projection_is_the_matrix_product(oracle):
    """Random BF16 inputs: equal, after one rounding, to the float64 matrix
    product of the decoded values (numpy's routine, not the oracle's loop)."""
    g = torch.Generator().manual_seed(2)
    x = torch.randn((5, 96), generator=g).to(torch.bfloat16)
    w = torch.randn((7, 96), generator=g).to(torch.bfloat16)
    want = (x.double().numpy() @ w.double().numpy().T).astype(np.float32)
    got = oracle.indexer_project(x.view(torch.int16).numpy().view(np.uint16),
                                 w.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(got, want)


def _pages(num_pages, D_I, dt):
    if dt == "f32":
        return np.full((num_pages, 16, D_I), 7.0, np.float32)
    return np.full((num_pages, 16, D_I), 0x40E0, np.uint16)     # 7.0 in BF16


def test_compression_mean_pooling_and_selection(oracle):
    """wphi = [I/4, I/4, I/4, I/4] pools the group's four token keys into their
    mean; wphi = [0, I, 0, 0] selects the second token's key; a bias adds."""
    D_I = 8
    rng = np.random.default_rng(3)
    k_tok = rng.integers(-8, 8, size=(3, 4, D_I)).astype(np.float32)   # small integers: exact sums
    I = np.eye(D_I, dtype=np.float32)
    pt = np.array([[2, 0, 1]], np.int32)
    gid = np.array([0, 17, 40], np.int32)     # logical pages 0, 1, 2 -> physical 2, 0, 1
    mean_w = np.concatenate([I / 4] * 4, axis=1)
    pages = _pages(3, D_I, "f32")
    assert oracle.compress_keys(k_tok, gid, mean_w, pages, pt) == 0
    assert np.array_equal(pages[2, 0], k_tok[0].mean(axis=0))
    assert np.array_equal(pages[0, 1], k_tok[1].mean(axis=0))
    assert np.array_equal(pages[1, 8], k_tok[2].mean(axis=0))
    sel_w = np.concatenate([0 * I, I, 0 * I, 0 * I], axis=1)
    bias = np.arange(D_I, dtype=np.float32)
    assert oracle.compress_keys(k_tok, gid, sel_w, pages, pt, bias=bias) == 0
    assert np.array_equal(pages[2, 0], k_tok[0, 1] + bias)
    assert np.array_equal(pages[1, 8], k_tok[2, 1] + bias)


def test_compression_writes_only_its_rows(oracle):
    """Each group lands in row g % 16 of page table[req][g // 16]; every other
    row keeps its contents; out-of-range requests and pages are skipped."""
    D_I = 4
    k_tok = np.ones((4, 4, D_I), np.float32)
    wphi = np.concatenate([np.eye(D_I, dtype=np.float32)] * 4, axis=1)   # sum of the four keys
    pt = np.array([[1, 3], [0, 99]], np.int32)
    gid = np.array([5, 16, 18, 20], np.int32)
    req = np.array([0, 0, 1, 1], np.int32)    # (1, 18) and (1, 20) -> page 99: out of range
    pages = _pages(4, D_I, "f32")
    before = pages.copy()
    assert oracle.compress_keys(k_tok, gid, wphi, pages, pt, g_req=req) == 2
    written = {(1, 5), (3, 0)}
    for p in range(4):
        for r in range(16):
            if (p, r) in written:
                assert np.all(pages[p, r] == 4.0)
            else:
                assert np.array_equal(pages[p, r], before[p, r])


def test_compression_bf16_storage_rounds_to_nearest_even(oracle):
    """BF16 storage keeps 8 significant bits: 1 + 2^-8 is a tie and rounds to
    1 (even), 1 + 3 * 2^-9 rounds up to 1 + 2^-7, -(2 + 2^-6) is exact."""
    D_I = 4
    k_tok = np.zeros((1, 4, D_I), np.float32)
    k_tok[0, 0] = [1 + 2.0 ** -8, 1 + 3 * 2.0 ** -9, -(2 + 2.0 ** -6), 0.5]
    wphi = np.concatenate([np.eye(D_I, dtype=np.float32)] + [np.zeros((D_I, D_I), np.float32)] * 3, axis=1)
    pages = _pages(1, D_I, "bf16")
    oracle.compress_keys(k_tok, np.array([3], np.int32), wphi, pages, np.zeros((1, 1), np.int32))
    got = torch.from_numpy(pages[0, 3].view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    assert list(got) == [1.0, 1 + 2.0 ** -7, -(2 + 2.0 ** -6), 0.5]
