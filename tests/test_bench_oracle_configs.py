"""The bench's host-only oracle mode (`--impl reference --oracle-configs`) on
shrunken stand-ins of the configs: one line listing every config, each with
an every-core and a one-core rate, and the prefill chunk both sampled and,
when asked, whole."""
import argparse
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_oracle_configs_line(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    from indexer_top_sparse_c4_b200 import workloads as wl
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    real_make = wl.make
    small = dict(B=2, ctx=2048, Hq=4, Hkv=1, D=64, H_I=2, D_I=32, kv_dtype="fp8", q_dtype="bf16",
                 dist="peaked", pages="perm")
    monkeypatch.setattr(wl, "b1_16k", lambda seed=0: wl.tiny(seed=seed, K=16))
    monkeypatch.setattr(wl, "b8_262k", lambda K=512, seed=0: real_make("b8_small", K=K, seed=seed, device="cpu",
                                                                        **small))
    monkeypatch.setattr(wl, "prefill_chunk", lambda seed=0: wl.tiny(seed=seed))
    monkeypatch.setattr(wl, "SWEEP_CASES", ((4096, 1, (4, 1), 512, "bf16", "ties"),))
    monkeypatch.setattr(wl, "sweep_case", lambda ctx, B, heads, K, kv, dist, seed=0: wl.tiny(seed=seed, K=8))
    args = argparse.Namespace(seed=0, cpu_seconds=0.1, oracle_full_prefill=True)
    line = bench.oracle_configs_arm(args)
    assert line["impl"] == "reference" and line["host_cores"] == (os.cpu_count() or 1)
    rows = line["oracle_configs"]
    names = [r["workload"] for r in rows]
    assert names[2:5] == ["b8_decode_262k_fp8_k512", "b8_decode_262k_fp8_k1024", "b8_decode_262k_fp8_k2048"]
    assert len(rows) == 2 + 3 + 2 + 1                  # tiny, B1, B8 x 3, prefill sampled + whole, sweep
    for r in rows:
        assert r["all_cores"]["tokens_per_s"] > 0 and r["all_cores"]["steps"] >= 1
    assert all("one_core" in r for i, r in enumerate(rows) if i != 6)
    assert "one_core" not in rows[6]                    # the whole prefill chunk: every core only
