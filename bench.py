"""Benchmark of the QSA decode hot path on B200: B8 x 262,144-token FP8 KV.

One step = one layer's decode of 8 requests through all four stages of
libqsa.so in three launches (indexer scores -> Top-K groups expanded to tokens ->
sparse attention),
inputs resident in HBM.  Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--budget 512]
    python bench.py --impl reference      # the CPU oracle, timed on host cores

Timing: CUDA events on the launching stream, W untimed warm-up steps, K timed
steps between a barrier + synchronize on both sides, max over ranks.  Two
independent input sets alternate between steps; each step streams 256 MiB of
indexer keys (twice the 126 MB L2), so no step finds its inputs in L2.
Multi-GPU (torchrun): every rank runs its own batch of 8 requests (weak
scaling); ranks exchange nothing on the data path.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QSA sparse-decode tokens/s @B8×262K FP8 KV; achieved HBM GB/s vs B200 peak"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # the B200's nominal HBM3e bandwidth, reported beside the measured peak
KERNELS_PER_STEP = 3  # index, Top-K with expansion, attention (partials merged inside the clusters)


def peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic(context):
    """DRAM bytes per full-size launch of the indexer scan, from the figure
    committed beside its ncu summary (profiles/*.json), or None when the
    kernel source changed since it was captured (or the workload is not the
    262,144-token one the figure is scaled to)."""
    import hashlib
    if context != 262144:
        return None
    try:
        with open(os.path.join(ROOT, "profiles", "index_scores_b8_decode_65536_fp8.json")) as f:
            rec = json.load(f)
        src = open(os.path.join(ROOT, rec["source_file"]), "rb").read()
        if hashlib.sha256(src).hexdigest()[:16] != rec["source_sha256_16"]:
            return None
        return int(rec["traffic_full_size_bytes_per_launch"])
    except Exception:
        return None


def algorithmic_bytes(w, n_tok_total):
    """Algorithmic bytes of one step (the headline metric's definition):
    every candidate group's compressed key, plus the K and V rows of every
    selected token for every KV head."""
    kv_elem = {"fp8": 1, "bf16": 2, "f32": 4}[w.kv_dtype]
    idx_elem = w.k_idx_pages.element_size()
    groups = int((w.q_pos // 4).sum().item())
    idx_bytes = groups * w.D_I * idx_elem
    kv_bytes = n_tok_total * w.Hkv * w.D * 2 * kv_elem
    return idx_bytes, kv_bytes


# ---- distributed plumbing ---------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(value: float, device) -> float:
    """Max of a host float over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def rank_seed(base: int, rank: int) -> int:
    return base + 1000 * rank


def weak_value(world: int, batch: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank decodes its own batch in each step."""
    return world * batch / (ms_per_step / 1e3)


# ---- clocks --------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        except Exception:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows)}


# ---- the GPU arm -----------------------------------------------------------------------

def make_sets(K, device, seed, n_sets=2, context=262144):
    from indexer_top_sparse_c4_b200 import workloads as wl
    from indexer_top_sparse_c4_b200.pipeline import QSAStep
    sets = []
    for i in range(n_sets):
        w = wl.b8_262k(K=K, device=device, seed=seed + i, ctx=context)
        sets.append(QSAStep(w))
    return sets


STAGES = ("index_scores", "select", "attention")
STAGE_NAMES = ("index_scores", "topk_expand", "sparse_attn_decode")


def capture(sets, steps, stages=STAGES):
    """One CUDA graph of `steps` consecutive QSA steps (alternating input
    sets), each step the given stages in order."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            st = sets[i % len(sets)]
            for name in stages:
                getattr(st, name)()
    return g


def replay_ms(g):
    """Device time of one replay of `g` (CUDA events on the current stream)."""
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    g.replay()
    end.record()
    torch.cuda.synchronize()
    barrier()
    return start.elapsed_time(end)


def time_steps(sets, steps, warmup, stream):
    """Device time (ms) of exactly `steps` steps replayed from one CUDA graph,
    after `warmup` eager steps and one untimed replay."""
    with torch.cuda.stream(stream):
        for i in range(warmup):
            sets[i % len(sets)].run()
        torch.cuda.synchronize()
        g = capture(sets, steps)
        g.replay()
        total = replay_ms(g)
    del g
    return total


def time_stages(sets, reps, stream):
    """Per-stage device times (us).  `alone`: a graph of `reps` launches of that
    stage only (for the indexer scan every launch streams its 256 MiB of keys
    from HBM, so this is its true launch duration).  The Top-K consumes the
    prefix histogram the scan leaves, so it is timed after the scan: the graph
    of (scan, Top-K) pairs minus the graph of scans.  `in_step`: what the stage
    adds to a step, i.e. the step graph minus the same graph without it."""
    def timed(stages):
        g = capture(sets, reps, stages)
        g.replay()
        ms = replay_ms(g)
        del g
        for st in sets:   # graphs without the Top-K leave the histogram counted up
            if st.prefix_hist is not None:
                st.prefix_hist.zero_()
        return ms

    alone, in_step = {}, {}
    with torch.cuda.stream(stream):
        t_full = timed(STAGES)
        for name in STAGES:
            if name == "select" and sets[0].prefix_hist is not None:
                alone[name] = (timed(("index_scores", "select")) - timed(("index_scores",))) / reps * 1e3
            else:
                alone[name] = timed((name,)) / reps * 1e3
            in_step[name] = (t_full - timed(tuple(x for x in STAGES if x != name))) / reps * 1e3
    return alone, in_step


def pack_inputs(st):
    """Rebind the step's per-step inputs (queries, indexer queries and weights,
    positions, request ids) to views of ONE device buffer, and return it with a
    pinned host twin holding the same bytes: a step's inputs then cross PCIe
    in a single copy.  Each view starts on a 256-byte boundary."""
    w = st.w
    names = ("q", "q_idx", "w_idx", "q_pos", "q_req")
    rebind_sel = st.sel_pos is w.q_pos
    offs, n = [], 0
    for nm in names:
        x = getattr(w, nm)
        offs.append(n)
        n += -(-x.numel() * x.element_size() // 256) * 256
    dev = torch.empty(n, dtype=torch.uint8, device=w.q.device)
    for nm, o in zip(names, offs):
        x = getattr(w, nm)
        nb = x.numel() * x.element_size()
        view = dev[o:o + nb].view(x.dtype).view(x.shape)
        view.copy_(x)
        setattr(w, nm, view)
    if rebind_sel:
        st.sel_pos = w.q_pos
    host = dev.cpu().pin_memory()
    return dev, host


def time_e2e(sets, steps, warmup, stream, graph=True):
    """Through the public API with host buffers: every step copies its
    query-side inputs from pinned host memory to the device (one packed
    copy), runs the calls and copies the output back to pinned host memory.
    The copies run on two copy streams, so step i+1's inputs go up and step
    i's output comes down while the kernels of step i (i+1) run; events keep
    each buffer safe (a set's inputs are overwritten only after the kernels
    that read them, its output only after its previous copy-out).  The KV
    cache and the indexer keys are resident device state.
    graph=True: the K timed steps are one captured CUDA graph (the calls'
    host work happens once, at capture).  graph=False: every step issues its
    copies and library calls from the host inside the timed region, the
    calls bound once by QSAStep.bind (their C argument checks and launches
    included, the Python argument conversion not)."""
    hosts = []
    for st in sets:
        if not hasattr(st, "_e2e_buffers"):
            dev, host = pack_inputs(st)
            st._e2e_buffers = (host, dev, torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory())
        hosts.append(st._e2e_buffers)
    h2d = hosts[0][1].numel()
    d2h = hosts[0][2].numel() * hosts[0][2].element_size()
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    n = len(sets)
    # eager: each step's library calls are bound once (QSAStep.bind) and
    # issued from the host every step; the graph captures run() itself
    bound = [st.bind(stream) for st in sets] if not graph else None

    def steps_on(main, count):
        ev_h = [torch.cuda.Event() for _ in range(count)]
        ev_k = [torch.cuda.Event() for _ in range(count)]
        ev_d = [torch.cuda.Event() for _ in range(count)]
        cin.wait_stream(main)
        cout.wait_stream(main)
        for i in range(count):
            st = sets[i % n]
            hin, dev_in, hout = hosts[i % n]
            with torch.cuda.stream(cin):
                if i >= n:
                    cin.wait_event(ev_k[i - n])   # the kernels that read this set's inputs are done
                dev_in.copy_(hin, non_blocking=True)
                ev_h[i].record(cin)
            main.wait_event(ev_h[i])
            if i >= n:
                main.wait_event(ev_d[i - n])      # this set's previous output has been copied out
            if bound is not None and main is stream:
                bound[i % n]()
            else:
                st.run(main)
            ev_k[i].record(main)
            with torch.cuda.stream(cout):
                cout.wait_event(ev_k[i])
                hout.copy_(st.out, non_blocking=True)
                ev_d[i].record(cout)
        main.wait_stream(cin)
        main.wait_stream(cout)

    with torch.cuda.stream(stream):
        steps_on(stream, warmup)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                steps_on(stream, steps)
            g.replay()
            torch.cuda.synchronize()
            barrier()
            a.record()
            g.replay()
            b.record()
        else:
            barrier()
            torch.cuda.synchronize()
            a.record()
            steps_on(stream, steps)
            b.record()
    torch.cuda.synchronize()
    barrier()
    if graph:
        del g
    return a.elapsed_time(b), h2d, d2h


def gpu_arm(args):
    ws, rank, local = dist_env()
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from indexer_top_sparse_c4_b200 import build
    if rank == 0 and not os.path.exists(build.LIB):
        build.build()
    barrier()
    stream = torch.cuda.Stream(device)
    sets = make_sets(args.budget, device, rank_seed(args.seed, rank), context=args.context)
    w0 = sets[0].w
    with ClockSampler(local) as clk:
        total_ms = time_steps(sets, args.steps, args.warmup, stream)
        alone, in_step = time_stages(sets, 40, stream)
        e2e_ms, h2d, d2h = time_e2e(sets, args.steps, args.warmup, stream, graph=True)
        e2e_eager_ms, _, _ = time_e2e(sets, args.steps, args.warmup, stream, graph=False)
    total_ms = reduce_max(total_ms, device)
    ms = total_ms / args.steps
    e2e_ms = reduce_max(e2e_ms, device)
    e2e_eager_ms = reduce_max(e2e_eager_ms, device)
    host_copy = sets[0].w.numpy() if (ws == 1 and not args.no_cpu_baseline) else None
    n_tok_total = int(sets[0].n_tok.sum().item())
    idx_bytes, kv_bytes = algorithmic_bytes(w0, n_tok_total)
    # other budgets, same workload shape, reported beside the headline
    budgets = {}
    if args.all_budgets:
        for K in (1024, 2048):
            if K == args.budget:
                continue
            del sets
            torch.cuda.empty_cache()
            sets = make_sets(K, device, rank_seed(args.seed, rank), context=args.context)
            t = time_steps(sets, max(3, args.steps // 2), args.warmup, stream)
            t = reduce_max(t, device) / max(3, args.steps // 2)
            nt = int(sets[0].n_tok.sum().item())
            ib, kb = algorithmic_bytes(sets[0].w, nt)
            peak, _ = peak_hbm()
            gbs = (ib + kb) / (t / 1e3) / 1e9
            budgets[str(K)] = {"tokens_per_s": round(ws * w0.B / (t / 1e3), 1), "ms_per_step": round(t, 4),
                               "step_hbm_gbs": round(gbs, 1), "step_hbm_frac": round(gbs / peak, 4),
                               "step_hbm_frac_nominal": round(gbs / NOMINAL_HBM_GBS, 4),
                               "bytes_per_step": ib + kb}
    if rank != 0:
        return None
    peak, peak_kind = peak_hbm()
    idx_ms = alone["index_scores"] / 1e3
    idx_gbs = idx_bytes / (idx_ms / 1e3) / 1e9
    step_gbs = (idx_bytes + kv_bytes) / (ms / 1e3) / 1e9
    value = weak_value(ws, w0.B, ms)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
        "data": "synthetic",
        "config": decode_config(w0.name, w0.B, args.context, w0.Hq, w0.Hkv, w0.D, w0.H_I, w0.D_I, w0.K, ws),
        "roofline": {"kernel": "index_scores", "bound": "hbm", "achieved": round(idx_gbs, 1),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(idx_gbs / peak, 4), "peak_nominal": NOMINAL_HBM_GBS,
                     "frac_nominal": round(idx_gbs / NOMINAL_HBM_GBS, 4),
                     "traffic": profiled_traffic(args.context),
                     "algorithmic_bytes_per_launch": idx_bytes,
                     "duration_us": round(alone["index_scores"], 2)},
        "step_hbm": {"achieved": round(step_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(step_gbs / peak, 4), "peak_nominal": NOMINAL_HBM_GBS,
                     "frac_nominal": round(step_gbs / NOMINAL_HBM_GBS, 4),
                     "bytes_per_step": idx_bytes + kv_bytes,
                     "indexer_key_bytes": idx_bytes, "selected_kv_bytes": kv_bytes},
        "attention_hbm": {"bytes_per_launch": kv_bytes,
                          "duration_us": round(alone["attention"], 2),
                          "achieved": round(kv_bytes / (alone["attention"] / 1e6) / 1e9, 1),
                          "frac": round(kv_bytes / (alone["attention"] / 1e6) / 1e9 / peak, 4)},
        "stages_us": {"alone": {n: round(alone[k], 2) for n, k in zip(STAGE_NAMES, STAGES)},
                      "in_step": {n: round(in_step[k], 2) for n, k in zip(STAGE_NAMES, STAGES)},
                      "note": "alone: CUDA-event duration per launch from a graph of launches of that "
                              "stage; in_step: the step graph minus the same graph without the stage "
                              "(a marginal cost, not a duration)"},
        "e2e": {"value": round(ws * w0.B / (e2e_ms / args.steps / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms / args.steps, 5),
                "how": "pinned host inputs up, calls, output down, every step; the timed steps "
                       "replayed from one CUDA graph"},
        "e2e_eager": {"value": round(ws * w0.B / (e2e_eager_ms / args.steps / 1e3), 1),
                      "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "ms_per_step": round(e2e_eager_ms / args.steps, 5),
                      "how": "as e2e, but every step's copies and qsa_* calls are issued from the "
                             "host inside the timed region (no graph); the calls bound once by "
                             "QSAStep.bind, so the C argument checks and launches are timed and the "
                             "Python argument conversion is not"},
        "gpu_launches": (KERNELS_PER_STEP + (1 if sets[0].ws_bytes else 0)) * args.steps,
        "clocks": clk.summary(),
    }
    if budgets:
        line["other_budgets"] = budgets
    if args.mtp and ws == 1:
        line["mtp"] = mtp_summary(device, stream, args.seed, 20)
    if args.prefill and ws == 1:
        line["prefill"] = prefill_summary(device, stream, args.seed, 3)
    if args.features and ws == 1:
        line["features"] = features_summary(device, stream, args.seed)
    if host_copy is not None:
        line["cpu_baseline"] = cpu_baseline(host_copy, w0, args.cpu_seconds)
    return line


def graph_us(fn, reps, stream):
    """Device time per call of fn(i), i < reps, from one CUDA graph of the
    reps calls (CUDA events on the graph's stream)."""
    with torch.cuda.stream(stream):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(reps):
                fn(i)
        g.replay()
        ms = replay_ms(g)
        del g
    return ms / reps * 1e3


def features_summary(device, stream, seed):
    """The entry points beyond the four-stage decode step, each timed on the
    device (graphs of launches): the guess-verify-refine Top-K, the indexer
    projection and C4 compressed-key write, the dense and sparse graph
    families of the sequence-length threshold, and sequence-sharded decode
    emulated on this one GPU."""
    from indexer_top_sparse_c4_b200 import qsa, workloads as wl
    from indexer_top_sparse_c4_b200.dcp import QSADcpDecode
    from indexer_top_sparse_c4_b200.pipeline import QSADecodeGraphs, QSAStep
    out = {}
    reps = 20
    # ---- Top-K on the B8 x 262,144 rows: GVR (no hint), radix without and with the scan's histogram
    topk = {}
    for K in (512, 2048):
        sets = [QSAStep(wl.b8_262k(K=K, device=device, seed=seed + i)) for i in (0, 1)]
        for st in sets:
            st.run()
        torch.cuda.synchronize()
        path = torch.empty((8,), dtype=torch.int32, device=device)
        g = graph_us(lambda i: qsa.qsa_topk_groups_gvr(sets[i % 2].scores, sets[i % 2].w.q_pos, K, sets[i % 2].sel,
                                                      sets[i % 2].n_sel, path=path), reps, stream)
        r = graph_us(lambda i: qsa.qsa_topk_groups(sets[i % 2].scores, sets[i % 2].w.q_pos, K, sets[i % 2].sel,
                                                   sets[i % 2].n_sel), reps, stream)
        scan = graph_us(lambda i: sets[i % 2].index_scores(), reps, stream)
        both = graph_us(lambda i: (sets[i % 2].index_scores(), sets[i % 2].topk()), reps, stream)
        for st in sets:
            st.prefix_hist.zero_()
        topk[str(K)] = {"gvr_us": round(g, 2), "radix_no_hint_us": round(r, 2),
                        "radix_with_scan_histogram_us": round(both - scan, 2),
                        "gvr_paths": sorted(set(path.tolist()))}
        del sets
    out["topk_b8_262k"] = topk
    # ---- indexer projection and compressed-key write (hidden 5,120, 4 x 128 indexer)
    H, N, D_I = 5120, 4 * 128 + 4 + 128, 128
    w, wphi, bias = wl.indexer_weights(H, 4, D_I, seed=seed, device=device)
    proj = {}
    for T in (8, 8192):
        x = wl.hidden_states(T, H, seed=seed + 1, device=device)
        y = torch.empty((T, N), dtype=torch.float32, device=device)
        us = graph_us(lambda i: qsa.qsa_indexer_project(x, w, y), reps, stream)
        flop = 2.0 * T * H * N
        proj[str(T)] = {"us": round(us, 2), "tflops": round(flop / us / 1e6, 1),
                        "weight_gbs": round(N * H * 2 / us / 1e3, 1)}
    pages = torch.zeros((8192 // 64 + 1, 16, D_I), dtype=torch.float32, device=device)
    pt = torch.arange(pages.shape[0], dtype=torch.int32, device=device).view(1, -1)
    g_id = torch.arange(8192 // 4, dtype=torch.int32, device=device)
    cmp_us = graph_us(lambda i: qsa.qsa_compress_keys(y[:, 4 * 128 + 4:], g_id, wphi, pages, pt, bias=bias), reps,
                      stream)
    out["indexer_write"] = {"projection": proj, "bound": {"8": "hbm (the weights)", "8192": "tensor"},
                            "compress_2048_groups_us": round(cmp_us, 2)}
    # ---- graph families of the sequence-length threshold (B8, 16,384 context, threshold 6,000)
    pos = torch.full((8,), 16383, dtype=torch.int32)
    wt = wl.make("thr", B=8, ctx=16384, Hq=16, Hkv=2, D=256, H_I=4, D_I=128, K=512, kv_dtype="fp8",
                 q_dtype="bf16", dist="peaked", seed=seed, device=device, q_pos=pos, q_req=torch.arange(8))
    st = QSAStep(wt, seq_len_threshold=6000)
    fams = QSADecodeGraphs(st, stream)

    def replays_us(name, max_len):
        with torch.cuda.stream(fams.stream):
            fams.replay(max_len)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(reps):
                assert fams.replay(max_len) == name
            b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps * 1e3

    sparse_us = replays_us("sparse", 16384)
    wt.q_pos.fill_(5999)
    dense_us = replays_us("dense", 6000)
    out["seq_len_threshold"] = {"threshold": st.threshold, "sparse_family_step_us": round(sparse_us, 2),
                                "dense_family_step_us_at_6000_tokens": round(dense_us, 2)}
    del fams, st, wt
    # ---- sequence-sharded decode emulated on one GPU (all shards in turn, merges included)
    dcp = {}
    wd = wl.b8_262k(K=512, device=device, seed=seed)
    for R in (2, 4):
        d = QSADcpDecode(wd, R)
        us = graph_us(lambda i: d.run(), 5, stream)
        dcp[str(R)] = {"emulated_step_us": round(us, 2),
                       "records_bytes_per_rank": 8 * wd.K * 8, "partials_bytes_per_rank": 8 * 16 * 256 * 4 + 8 * 16 * 4}
        del d
    out["dcp_b8_262k_k512"] = {"shards": dcp, "note": "one GPU runs every shard in turn; no collective crosses "
                                                      "NVLink in this measurement"}
    torch.cuda.empty_cache()
    return out


# ---- the prefill chunk ------------------------------------------------------------------

def peak_bf16(sustained=False):
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained" if sustained else "bf16_tflops"]), "measured"
    except Exception:
        return (1400.0 if sustained else 1590.0), "fallback"


def prefill_summary(device, stream, seed, reps):
    """The prefill chunk (8,192 new query tokens after a 57,344-token prefix,
    24/2 heads of dim 256, BF16 KV, budget 512 groups) through the four stages.
    Each stage is timed alone from a CUDA graph of `reps` launches; the whole
    step likewise.  The dense indexer contraction is reported in TFLOP/s
    against the measured BF16 tensor peak (burst: each kernel is timed on its
    own); the attention, a gather of K/V rows that come from L2, by its
    gather rate (GB/s, and per SM), with its TFLOP/s beside it."""
    from indexer_top_sparse_c4_b200 import workloads as wl
    from indexer_top_sparse_c4_b200.pipeline import QSAStep
    w = wl.prefill_chunk(device=device, seed=seed)
    st = QSAStep(w, prefill=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            st.run()
        torch.cuda.synchronize()
        times = {}
        for name in STAGES + ("step",):
            g = capture([st], reps, STAGES if name == "step" else (name,))
            g.replay()
            times[name] = replay_ms(g) / reps
            del g
    # the Top-K alone on the chunk's scores: radix passes against the
    # guess-verify-refine mode (same selection; the step uses the radix kernel)
    from indexer_top_sparse_c4_b200 import qsa
    sel2, n2 = torch.empty_like(st.sel), torch.empty_like(st.n_sel)
    topk_radix_us = graph_us(lambda i: qsa.qsa_topk_groups(st.scores, st.sel_pos, w.K, sel2, n2), reps, stream)
    topk_gvr_us = graph_us(lambda i: qsa.qsa_topk_groups_gvr(st.scores, st.sel_pos, w.K, sel2, n2), reps, stream)
    sum_c = int((w.q_pos // 4).sum().item())
    sum_tok = int(st.n_tok.sum().item())
    idx_flop = 2.0 * w.H_I * w.D_I * sum_c
    attn_flop = 4.0 * w.D * w.Hq * sum_tok
    peak, kind = peak_bf16()
    idx_tf = idx_flop / (times["index_scores"] / 1e3) / 1e12
    attn_tf = attn_flop / (times["attention"] / 1e3) / 1e12
    # the attention is a gather: every (query, KV head) row reads its selected
    # K and V rows (2 x D x 2 bytes per token), almost all of them from L2
    gather_bytes = float(sum_tok) * w.Hkv * 2 * w.D * 2
    gather_gbs = gather_bytes / (times["attention"] / 1e3) / 1e9
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    names = dict(zip(STAGES, ("index_scores", "topk_expand", "sparse_attn_prefill")))
    return {
        "workload": w.name, "T": w.T, "context": int(w.q_pos.max().item()) + 1, "Hq": w.Hq, "Hkv": w.Hkv,
        "D": w.D, "budget_groups": w.K, "kv_storage": "bf16", "indexer_operands": "bf16",
        "query_tokens_per_s": round(w.T / (times["step"] / 1e3), 1),
        "ms_per_step": round(times["step"], 4),
        "stages_ms": {names[k]: round(times[k], 4) for k in STAGES},
        "topk_alone_ms": {"radix": round(topk_radix_us / 1e3, 4), "gvr": round(topk_gvr_us / 1e3, 4)},
        "index_scores": {"bound": "tensor", "flop_per_launch": idx_flop,
                         "achieved": round(idx_tf, 1), "peak": peak, "peak_kind": kind,
                         "unit": "TFLOP/s", "frac": round(idx_tf / peak, 4)},
        "sparse_attn_prefill": {"bound": "latency of L2 gathers", "bytes_per_launch": gather_bytes,
                                "achieved": round(gather_gbs, 1), "unit": "GB/s",
                                "per_sm_gbs": round(gather_gbs / sms, 1),
                                "note": "K/V rows gathered from L2 (93% hits); the committed ncu summary shows L2 "
                                        "throughput at 32% of its peak and issue at 49% with 12 warps per SM: "
                                        "no bandwidth roof is reached",
                                "tensor": {"flop_per_launch": attn_flop, "achieved": round(attn_tf, 1),
                                           "peak": peak, "peak_kind": kind, "unit": "TFLOP/s",
                                           "frac": round(attn_tf / peak, 4)}},
    }


def mtp_summary(device, stream, seed, loops, drafts=2):
    """The MTP draft loop with index sharing on the B8 x 262,144 FP8 workload:
    a capture step at p0 (the last token of a block) and `drafts` draft steps
    at p0 + 1 .. that reuse its selection (plus the group completed since)
    and only attend.  Two loop sets alternate, so every capture step streams
    its 256 MiB of indexer keys from HBM; `loops` loops are one CUDA graph."""
    from indexer_top_sparse_c4_b200 import workloads as wl
    from indexer_top_sparse_c4_b200.pipeline import QSADraftLoop
    ctx, B, K = 262144, 8, 512
    p0 = ((ctx - 4 - drafts) // 4) * 4 + 3   # the last token of a block; p0 + drafts < ctx
    sets = []
    for sd in (seed, seed + 1):
        w = wl.make(f"mtp_b8_262k_fp8_k{K}_draft{drafts}", B=B, ctx=ctx, Hq=16, Hkv=2, D=256, H_I=4,
                    D_I=128, K=K, kv_dtype="fp8", q_dtype="bf16", dist="peaked", pages="perm", seed=sd,
                    device=device, q_pos=torch.full((B,), p0, dtype=torch.int32),
                    q_req=torch.arange(B, dtype=torch.int32))
        sets.append(QSADraftLoop(w, drafts=drafts, seed=sd + 7))
    with torch.cuda.stream(stream):
        for i in range(4):
            sets[i % 2].run()
        torch.cuda.synchronize()
        times = {}
        for name in ("loop", "capture", "draft"):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(loops):
                    st = sets[i % 2]
                    if name == "loop":
                        st.run()
                    elif name == "capture":
                        st.capture.run()
                    else:
                        st.draft_step(0)
            g.replay()
            times[name] = replay_ms(g) / loops
            del g
        for st in sets:  # the capture-only graph leaves the histograms counted up
            st.capture.prefix_hist.zero_()
    ok = all(int(st.status.item()) == 0 for st in sets)
    per_loop = B * (1 + drafts)
    return {"workload": sets[0].w.name, "B": B, "context": ctx, "capture_pos": p0, "drafts": drafts,
            "tokens_per_loop": per_loop, "tokens_per_s": round(per_loop / (times["loop"] / 1e3), 1),
            "ms_per_loop": round(times["loop"], 5),
            "stages_us": {"capture_step": round(times["capture"] * 1e3, 2),
                          "draft_step": round(times["draft"] * 1e3, 2)},
            "device_status_ok": ok}


def prefill_arm(args):
    """`--workload prefill`: only the prefill chunk, one JSON line."""
    ws, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from indexer_top_sparse_c4_b200 import build
    if not os.path.exists(build.LIB):
        build.build()
    stream = torch.cuda.Stream(device)
    summary = prefill_summary(device, stream, args.seed, max(1, args.steps))
    return {"metric": "QSA prefill query tokens/s (8,192-token chunk, 65,536 context)",
            "value": summary["query_tokens_per_s"], "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": 3, "ms_per_step": summary["ms_per_step"],
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic", "prefill": summary}


# ---- the oracle on host cores ----------------------------------------------------------

def oracle_inputs(K, seed, context=262144):
    """Host copies of the B8 workload the GPU arm times (same generator, seed
    and recipe).  They are drawn on the GPU when there is one, which is
    where the GPU arm draws them, and copied to the host; the oracle then
    runs on the host cores only."""
    from indexer_top_sparse_c4_b200 import workloads as wl
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = wl.b8_262k(K=K, device=dev, seed=seed, ctx=context)
    n, k_scale, v_scale = w.numpy(), w.k_scale, w.v_scale
    del w
    if dev == "cuda":
        torch.cuda.empty_cache()
    return n, k_scale, v_scale


def run_oracle_step(orc, n, K, k_scale, v_scale):
    """One decode step of every request in `n` through the oracle's four stages."""
    return orc.qsa_step(n["q"], n["q_idx"], n["w_idx"], n["k_idx_pages"], n["k_pages"], n["v_pages"],
                        n["page_table"], n["q_pos"], K, k_scale, v_scale, q_req=n["q_req"])


def _time_oracle(orc, n, K, k_scale, v_scale, seconds, min_steps=1):
    t0 = time.perf_counter()
    steps = 0
    while True:
        run_oracle_step(orc, n, K, k_scale, v_scale)
        steps += 1
        el = time.perf_counter() - t0
        if el >= seconds and steps >= min_steps:
            return steps, el


def cpu_baseline(n, w, seconds):
    """The oracle as it stands, on the host cores, over the GPU arm's own
    workload (all 8 requests per step, copied to the host): once with its
    OpenMP loop over requests on every core it can use, once on one core."""
    import oracle as orc
    orc.build()
    T = int(n["q_pos"].shape[0])
    host_cores = os.cpu_count() or 1
    orc.set_max_threads(host_cores)
    threads = orc.threads_for(T)
    steps, el = _time_oracle(orc, n, w.K, w.k_scale, w.v_scale, seconds)
    orc.set_max_threads(1)
    s1, el1 = _time_oracle(orc, n, w.K, w.k_scale, w.v_scale, seconds / 2)
    orc.set_max_threads(host_cores)
    return {"value": round(T * steps / el, 3), "unit": "tokens/s", "cores": threads,
            "host_cores": host_cores, "kind": "oracle",
            "sample": f"{steps} decode step(s) of all {T} requests of the GPU arm's workload "
                      f"(262,144 context, K={w.K} groups), all four stages, {el:.1f} s; the oracle's "
                      f"OpenMP loop runs over requests, so it uses min({T}, host cores) threads",
            "single_core": {"value": round(T * s1 / el1, 3), "unit": "tokens/s", "cores": 1,
                            "sample": f"{s1} step(s), {el1:.1f} s"}}


def decode_config(name, B, context, Hq, Hkv, D, H_I, D_I, K, ws):
    """The workload description both arms print."""
    return {"workload": name, "B": B, "context": context, "Hq": Hq, "Hkv": Hkv, "D": D, "H_I": H_I,
            "D_I": D_I, "budget_groups": K, "kv_storage": "fp8_e4m3 per-tensor scale",
            "indexer_keys": "fp32, peaked (5% +3 sigma)", "page_table": "random permutation, page size 64",
            "l2": "inputs larger than L2: 256 MiB of indexer keys per step, 2 alternating input sets",
            "parallelism": f"dp{ws} (independent request batches)"}


def reference_arm(args):
    """The oracle on the host cores: each timed step is one decode step of all
    8 requests of the workload the GPU arm times (same generator and seed)."""
    ws, rank, local = dist_env()
    if rank != 0:
        return None
    import oracle as orc
    orc.build()
    host_cores = os.cpu_count() or 1
    orc.set_max_threads(host_cores)
    n, k_scale, v_scale = oracle_inputs(args.budget, rank_seed(args.seed, 0), args.context)
    T = int(n["q_pos"].shape[0])
    for _ in range(args.warmup):
        run_oracle_step(orc, n, args.budget, k_scale, v_scale)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run_oracle_step(orc, n, args.budget, k_scale, v_scale)
    el = time.perf_counter() - t0
    value = T * args.steps / el
    threads = orc.threads_for(T)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": decode_config(f"b8_decode_{args.context // 1024}k_fp8_k{args.budget}", T, args.context,
                                16, 2, 256, 4, 128, args.budget, ws),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": threads,
                         "host_cores": host_cores, "kind": "oracle",
                         "sample": f"each step: all {T} requests ({args.context:,} context, "
                                   f"K={args.budget} groups), all four stages; the oracle's OpenMP "
                                   f"loop runs over requests"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def oracle_configs_arm(args):
    """`--impl reference --oracle-configs`: the oracle as it stands on the host
    cores, over every config: tiny, B1 16K, B8 262K at the three budgets, the
    prefill chunk (64 of its query rows; with --oracle-full-prefill also all
    of them, once, on every core) and the sweep's covering cases.  Each is
    timed with the oracle's OpenMP loop over query rows on every core it can
    use, and on one core, each for about --cpu-seconds / 4.  Host work only
    (the inputs are drawn on the host); one JSON line, a reported baseline."""
    ws, rank, local = dist_env()
    if rank != 0:
        return None
    import numpy as np
    import oracle as orc
    from indexer_top_sparse_c4_b200 import workloads as wl
    orc.build()
    host_cores = os.cpu_count() or 1
    secs = max(args.cpu_seconds / 4, 0.5)
    per_row = ("q", "q_idx", "w_idx", "q_pos", "q_req", "capture_pos")

    def rows_of(n, idx):
        m = dict(n)
        for k in per_row:
            if m.get(k) is not None:
                m[k] = np.ascontiguousarray(m[k][idx])
        return m

    def time_config(w, n, K, sample, name=None, modes=(("all_cores", None), ("one_core", 1))):
        T = int(n["q_pos"].shape[0])
        out = {"workload": name or w.name, "K": K, "rows": T, "threads": min(orc.threads_for(T), host_cores),
               "sample": sample}
        for label, threads in modes:
            threads = threads or host_cores
            orc.set_max_threads(threads)
            steps, el = _time_oracle(orc, n, K, w.k_scale, w.v_scale, secs)
            out[label] = {"tokens_per_s": round(T * steps / el, 3), "steps": steps, "seconds": round(el, 2)}
        orc.set_max_threads(host_cores)
        return out

    res = []
    for make in (lambda: wl.tiny(seed=args.seed), lambda: wl.b1_16k(seed=args.seed)):
        w = make()
        res.append(time_config(w, w.numpy(), w.K, "every query row, all four stages"))
    w = wl.b8_262k(K=2048, seed=args.seed)   # the budgets share the inputs; W fits K = 2,048
    n = w.numpy()
    for K in (512, 1024, 2048):
        res.append(time_config(w, n, K, "every query row (8), all four stages", f"b8_decode_262k_fp8_k{K}"))
    del w, n
    w = wl.prefill_chunk(seed=args.seed)
    n = w.numpy()
    idx = np.unique(np.linspace(0, w.T - 1, 64).astype(int))
    res.append(time_config(w, rows_of(n, idx), w.K,
                           f"{idx.size} of the {w.T:,} query rows, evenly spaced, all four stages"))
    if args.oracle_full_prefill:   # once, on every core (one core would take about half an hour)
        res.append(time_config(w, n, w.K, f"every query row ({w.T:,}), all four stages, once",
                               modes=(("all_cores", None),)))
    del w, n
    for case in wl.SWEEP_CASES:
        ctx, B, heads, K, kv, dist = case
        w = wl.sweep_case(ctx, B, heads, K, kv, dist, seed=ctx + B)
        res.append(time_config(w, w.numpy(), K, "every query row, all four stages"))
        del w
    return {"impl": "reference", "oracle_configs": res, "host_cores": host_cores, "kind": "oracle",
            "unit": "tokens/s (query rows through all four stages per second)",
            "note": "inputs drawn on the host (the same recipe and seeds; the GPU arm draws on the GPU)"}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--budget", type=int, default=512, help="budget in groups (512, 1024, 2048)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--context", type=int, default=262144,
                    help="tokens per request; smaller values give the small cases used for profiling")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--all-budgets", action="store_true", default=True)
    ap.add_argument("--headline-only", dest="all_budgets", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-mtp", dest="mtp", action="store_false",
                    help="skip the MTP draft loop (index sharing) line")
    ap.add_argument("--no-features", dest="features", action="store_false",
                    help="leave out the timings of the entry points beyond the decode step")
    ap.add_argument("--no-prefill", dest="prefill", action="store_false",
                    help="leave out the prefill-chunk summary of the decode line")
    ap.add_argument("--workload", choices=["decode", "prefill"], default="decode",
                    help="prefill: time only the 8,192-token prefill chunk (one GPU)")
    ap.add_argument("--oracle-configs", action="store_true",
                    help="with --impl reference: time the oracle on every config (host only)")
    ap.add_argument("--oracle-full-prefill", action="store_true",
                    help="with --oracle-configs: also every query row of the prefill chunk, once")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        line = oracle_configs_arm(args) if args.oracle_configs else reference_arm(args)
    elif args.workload == "prefill":
        line = prefill_arm(args)
    else:
        line = gpu_arm(args)
    if line is not None:
        print(json.dumps(line), flush=True)
    try:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()
    except Exception:
        pass


if __name__ == "__main__":
    main()
