"""Throughput of query-aware page-sparse decode over a paged KV cache on B200.

One step = one decode step of a 32-layer model with Llama-3.1-8B attention geometry
(batch 8, 32 query / 8 KV heads, head dim 128, 32768 tokens per sequence, page 16,
token budget 2048 = sink 64 + window 512 + top-k).  Per layer, one sa_sparse_decode call
scores every page against the query (streaming kernel, which also refreshes the summary
of each sequence's newest page from K), selects the top pages (per-pair select kernel)
and runs split-KV attention over the gathered pages (attention kernel plus the merge
kernel of the pairs split across warps).  Its two halves, sa_select_pages and
sa_attend_selected, are timed apart for context.  Every layer owns its own KV pool, so a
step touches ~4.3 GB (> L2) and nothing is served from L2 across layers.

The default llama32k run also times llama128k (131072 tokens per sequence), ragged
(4 sequences of 64K-256K tokens, page 32) and mla (latent 576/512, 128 query heads) the
same way over 8 layer pools each and adds their microseconds per layer-call and HBM
fractions to the line's config, and every grouped-query run adds the same step as one
persistent launch per layer (sa_sparse_decode_fused, single_launch_us_per_layer)
(--no-extras skips them).  cpu_baseline is the CPU oracle
on every host core (independent sequences on threads), its single-thread rate beside it.

Metric: sparse-decode seq*heads/s = (sequence, query head) attention outputs of one
layer-call per second, whole job.  The headline is timed on a CUDA graph of the step
with no event inside it; a second graph with an event between the two halves of every
layer gives the per-phase times behind "roofline" (events between kernels cost the
programmatic overlap of neighbouring kernels, so that pass is slightly slower).

  python bench.py [--gpus N] [--steps K] [--warmup W]
                  [--workload llama32k|llama128k|ragged|mla|prune|tiny]
  python bench.py --select-every 4   (cross-layer reuse: select at every 4th layer only)
  python bench.py --summaries fp8    (fp8 summaries rounded outward, sa_sparse_decode_fp8)
  python bench.py --impl reference ...   (the CPU oracle on a bounded sample)

Under torchrun (N > 1) every rank runs its own batch on its own GPU (weak scaling,
no collective on the data path); the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

N_LAYERS = 32
WORKLOADS = ("llama32k", "llama128k", "ragged", "mla", "tiny", "prune")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama32k", choices=WORKLOADS)
    ap.add_argument("--layers", type=int, default=None,
                    help="layer pools per step (default 32 for llama32k, 8 otherwise)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-extras", dest="extras", action="store_false",
                    help="llama32k: skip the llama128k / ragged / mla measurements that the "
                         "default run adds to the line's config")
    ap.add_argument("--seed", type=int, default=0,
                    help="offset added to the workload's seed (every rank adds its own)")
    ap.add_argument("--summaries", default="bf16", choices=["bf16", "fp8"],
                    help="fp8: page summaries as E4M3 records rounded outward "
                         "(sa_sparse_decode_fp8); grouped-query workloads only")
    ap.add_argument("--select-every", type=int, default=1,
                    help="cross-layer selection reuse: select pages at every R-th layer and "
                         "attend over that selection at the R-1 layers after it (default 1: "
                         "every layer selects its own pages)")
    return ap.parse_args()


def _json_default(o):
    if hasattr(o, "item"):
        return o.item()
    return str(o)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------------------------------
# algorithmic bytes (inherent to the method; workspace traffic excluded)
# ------------------------------------------------------------------------------------

def rank_seed(workload, rank, offset=0):
    """Seed of rank `rank`'s batch: every rank decodes its own sequences (replicas)."""
    return synth.WORKLOADS[workload]["seed"] + offset + 1000 * rank


def max_over_ranks(x, dist, device="cpu"):
    """The largest of the ranks' values of `x` (a duration): the job ends with its slowest
    rank.  `dist` is torch.distributed (or None for one process)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step, world, ms_per_step):
    """Units per second of the whole job: every rank processes its own units per step."""
    return units_per_rank_step * world / (ms_per_step * 1e-3)


def layer_bytes(geom, seq_lens, sel_count, P, fp8=False):
    """Per layer-call: (select_bytes, attend_bytes, update_bytes).  fp8: summaries are
    records of 2*Dk + 16 bytes per (page, KV head) instead of 4*Dk."""
    g = geom
    rec = 2 * g.Dk + 16 if fp8 else 4 * g.Dk
    nb = (seq_lens.astype(np.int64) + P - 1) // P
    summ = int(nb.sum()) * g.Hkv * rec
    pt = int(nb.sum()) * 4
    q = g.B * g.Hq * g.Dk * 2
    sel_bytes = summ + pt + q
    # valid tokens of the selected pages: every selected page is full except a
    # sequence's last page (always selected when the sequence is non-empty)
    tok = 0
    for b in range(g.B):
        L = int(seq_lens[b])
        last_valid = L - (nb[b] - 1) * P if nb[b] else 0
        for h in range(g.Hkv):
            c = int(sel_count[b, h])
            tok += c * P - (P - last_valid if c else 0)
    kv = tok * (g.Dk + (0 if g.v_aliases_k else g.Dv)) * 2
    att_bytes = kv + q + g.B * g.Hq * (g.Dv * 4 + 4)
    upd = g.B * g.Hkv * (P * g.Dk * 2 + rec)
    return sel_bytes, att_bytes, upd


# ------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in open(self.path):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------
# CPU oracle arm (cpu_baseline and --impl reference)
# ------------------------------------------------------------------------------------

def oracle_sample(case, seconds, select_every=1, fp8=False):
    """Time the CPU oracle's decode step (score + select + attend) sequence by sequence
    on the bench's own layer-0 data until ~`seconds` have elapsed.  With select_every=R
    the (sequence, layer) call of layer l scores and selects only when l % R == 0 and
    otherwise attends over the sequence's last selection.  fp8: scores over the fp8
    records."""
    import oracle
    g = case.geom
    if fp8:
        summ = oracle.page_summaries_fp8(g, case.k_cache, case.page_table, case.seq_lens)
        scorer = oracle.page_scores_fp8
    else:
        summ = oracle.page_summaries(g, case.k_cache, case.page_table, case.seq_lens)
        scorer = oracle.page_scores
    done, t_total = 0, 0.0
    b = 0
    last = {}
    while t_total < seconds:
        sub = synth.Geometry(1, g.Hq, g.Hkv, g.Dk, g.Dv, g.P, g.max_pages, g.n_pool, g.v_aliases_k)
        q = case.q[b:b + 1]
        pt = case.page_table[b:b + 1]
        sl = case.seq_lens[b:b + 1]
        layer = done // g.B
        t0 = time.perf_counter()
        if layer % select_every == 0 or b not in last:
            sc = scorer(sub, q, summ, pt, sl)
            last[b] = oracle.select_pages(sub, sc, sl, case.budget, case.sink, case.window)
        sel, cnt = last[b]
        oracle.attend(sub, q, case.k_cache, case.v_cache, pt, sl, sel, cnt, case.scale)
        t_total += time.perf_counter() - t0
        done += 1
        b = (b + 1) % g.B
    units = done * g.Hq
    return units / t_total, done, t_total


def oracle_sample_mt(case, seconds, select_every=1, fp8=False, threads=None):
    """oracle_sample on `threads` host threads at once (default: every core), each on its
    own sequences (thread i takes sequences i, i + threads, ...): the C oracle releases
    the GIL while it computes, so independent sequences run in parallel.  Returns
    (units per second of wall time, calls done, wall seconds, threads)."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    threads = threads or os.cpu_count() or 1
    threads = max(1, min(threads, case.geom.B))
    oracle.load()  # build/load once, before the threads start

    def worker(i):
        sub = dataclass_slice(case, i, threads)
        _, done, _ = oracle_sample(sub, seconds, select_every, fp8)
        return done

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        dones = list(ex.map(worker, range(threads)))
    wall = time.perf_counter() - t0
    done = sum(dones)
    return done * case.geom.Hq / wall, done, wall, threads


def dataclass_slice(case, i, step):
    """The decode case restricted to sequences i, i + step, ... (same pool)."""
    import dataclasses
    idx = np.arange(i, case.geom.B, step)
    g = dataclasses.replace(case.geom, B=len(idx))
    return dataclasses.replace(case, geom=g, q=case.q[idx], page_table=case.page_table[idx],
                               seq_lens=case.seq_lens[idx])


def workload_config(case, args, layers):
    """The workload description shared by the native and the reference lines."""
    g = case.geom
    fp8 = args.summaries == "fp8"
    R = args.select_every
    return {
        "workload": args.workload,
        "batch": g.B, "q_heads": g.Hq, "kv_heads": g.Hkv, "head_dim": g.Dk,
        "seq_len": int(case.seq_lens.max()), "page": g.P, "budget_tokens": case.budget,
        "sink": case.sink, "window": case.window, "layers_per_step": layers,
        "select_every": R,
        "summaries": "fp8 e4m3 rounded outward" if fp8 else "bf16",
        "call": ("sa_sparse_decode_fp8" if fp8 else "sa_sparse_decode") if R == 1 else
                "sa_select_pages + sa_attend_selected",
    }


def selection_counts(case):
    """Pages every (sequence, KV head) selects: min(ceil(len / P), budget / P), as the
    library's selection does by construction."""
    g = case.geom
    nb = (np.asarray(case.seq_lens, dtype=np.int64) + g.P - 1) // g.P
    k = np.minimum(nb, case.budget // g.P).astype(np.int32)
    return np.repeat(k[:, None], g.Hkv, axis=1)


def step_bytes_of(case, args, layers, sel_count):
    """Algorithmic bytes of one step: attention every layer, scoring and selection (with
    the newest pages' refresh) every select_every layers."""
    sel_b, att_b, upd_b = layer_bytes(case.geom, case.seq_lens, sel_count, case.geom.P,
                                      args.summaries == "fp8")
    R = args.select_every
    return layers * att_b + ((layers + R - 1) // R) * (sel_b + upd_b)


def run_config(case, args, layers, world, step_bytes):
    """workload_config plus the run's L2 and parallelism description, worded as the
    native line words them."""
    return {
        **workload_config(case, args, layers),
        "l2": "inputs larger than L2: %d distinct layer pools, %.2f GB touched per step"
              % (layers, step_bytes / 1e9),
        "parallelism": "replicas (batch split), no collective" if world > 1 else "1 GPU",
        "algorithmic_bytes_per_layer": step_bytes / layers,
    }


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    if args.workload == "prune":
        pc = synth.prune_case("prune", seed=rank_seed("prune", 0, args.seed))
        v, done, t = oracle_prune_sample(pc, args.cpu_seconds)
        print(json.dumps({
            "impl": "reference", "metric": "sessions compacted/s", "value": v,
            "unit": "sessions compacted/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "ms_per_step": None,
            "config": {"workload": "prune"},
            "cpu_baseline": {"value": v, "unit": "sessions compacted/s", "cores": 1,
                             "kind": "oracle",
                             "sample": "%d sessions compacted, %.1f s" % (done, t)},
            "e2e": {"value": v, "unit": "sessions compacted/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}, default=_json_default), flush=True)
        return 0
    case = synth.decode_case(args.workload, seed=rank_seed(args.workload, 0, args.seed))
    v, done, t, cores = oracle_sample_mt(case, args.cpu_seconds, args.select_every,
                                         args.summaries == "fp8")
    line = {
        "impl": "reference", "metric": "sparse-decode seq*heads/s", "value": v,
        "unit": "seq*heads/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "ms_per_step": None,
        "config": run_config(case, args, args.layers, world,
                             step_bytes_of(case, args, args.layers, selection_counts(case))),
        "cpu_baseline": {"value": v, "unit": "seq*heads/s", "cores": cores, "kind": "oracle",
                         "sample": "%d (sequence, layer) decode calls of layer 0 "
                                   "(score+select%s, attend; all %d heads) on %d host "
                                   "threads, %.1f s wall" % (
                                       done, "" if args.select_every == 1 else
                                       " every %d layers" % args.select_every,
                                       case.geom.Hq, cores, t)},
        "e2e": {"value": v, "unit": "seq*heads/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line, default=_json_default), flush=True)
    return 0


# ------------------------------------------------------------------------------------
# native arm
# ------------------------------------------------------------------------------------

def run_native(args, rank, world, dist):
    import torch
    import paged_kv_cache_sa_b200 as sa
    from paged_kv_cache_sa_b200 import Geometry

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    hbm_peak, _, peak_kind = peaks()

    # ---- inputs: layer 0 from the seeded generator (rank-specific seed), other layers
    # are the same bytes rolled along the page axis (distinct memory and content)
    case = synth.decode_case(args.workload, seed=rank_seed(args.workload, rank, args.seed))
    g = Geometry.of(case.geom)
    P = g.P
    F8 = args.summaries == "fp8"
    if F8 and (g.v_aliases_k or args.select_every != 1):
        raise SystemExit("--summaries fp8 needs a grouped-query workload and --select-every 1")
    L_layers = args.layers
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16
                                                          else a)).to(dev)
    k0 = t(case.k_cache)
    v0 = t(case.v_cache) if case.v_cache is not None else None  # latent: V aliases K
    pt, sl = t(case.page_table), t(case.seq_lens)
    rng = np.random.default_rng(1234 + rank)
    ks, vs, qs, summs = [], [], [], []
    stride = max(1, g.n_pool // L_layers)
    for l in range(L_layers):
        ks.append(k0 if l == 0 else torch.roll(k0, shifts=l * stride, dims=0))
        vs.append(None if v0 is None else
                  (v0 if l == 0 else torch.roll(v0, shifts=l * stride, dims=0)))
        qn = case.q if l == 0 else synth.f32_to_bf16(rng.standard_normal(case.q.shape).astype(np.float32))
        qs.append(t(qn))
        if F8:
            summs.append(sa.empty_summaries_fp8(g, dev))
            sa.page_summaries_fp8(g, ks[l], pt, sl, summs[l])
        else:
            summs.append(torch.empty((g.n_pool, g.Hkv, 2, g.Dk), dtype=torch.int16, device=dev))
            sa.page_summaries(g, ks[l], pt, sl, summs[l])
    # per-page summaries (row a-1) of one layer's pool, timed alone: K read once
    e_s0, e_s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e_s0.record()
    for _ in range(3):
        if F8:
            sa.page_summaries_fp8(g, ks[0], pt, sl, summs[0])
        else:
            sa.page_summaries(g, ks[0], pt, sl, summs[0])
    e_s1.record()
    torch.cuda.synchronize()
    summ_ms = e_s0.elapsed_time(e_s1) / 3
    n_used = int(((case.seq_lens.astype(np.int64) + P - 1) // P).sum())
    summ_bytes = int(case.seq_lens.astype(np.int64).sum()) * g.Hkv * g.Dk * 2 + \
        n_used * g.Hkv * (2 * g.Dk + 16 if F8 else 4 * g.Dk) + n_used * 4
    K = case.budget // P
    ws = sa.Workspace.for_decode(g, case.budget)
    sel = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device=dev)
    cnt = torch.empty((g.B, g.Hkv), dtype=torch.int32, device=dev)
    phys = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device=dev)
    outs = [torch.empty((g.B, g.Hq, g.Dv), dtype=torch.float32, device=dev) for _ in range(L_layers)]
    lses = [torch.empty((g.B, g.Hq), dtype=torch.float32, device=dev) for _ in range(L_layers)]
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
          for _ in range(L_layers)]

    R = args.select_every

    def step_fused():
        # the headline: one sa_sparse_decode per layer (selection + attention)
        if F8:
            for l in range(L_layers):
                sa.sparse_decode_fp8(g, qs[l], ks[l], vs[l], summs[l], pt, sl, case.budget,
                                     case.sink, case.window, case.scale, ws, out=outs[l],
                                     lse=lses[l], sel_out=sel, sel_count_out=cnt,
                                     n_tail_refresh=1)
            return
        if R == 1:
            for l in range(L_layers):
                sa.sparse_decode(g, qs[l], ks[l], vs[l], summs[l], pt, sl, case.budget,
                                 case.sink, case.window, case.scale, ws, out=outs[l],
                                 lse=lses[l], sel_out=sel, sel_count_out=cnt, n_tail_refresh=1)
            return
        # cross-layer reuse: layer l selects when l % R == 0; the layers after it attend
        # over that selection (physical pages of the shared page table) with their own
        # query, keys and values
        for l in range(L_layers):
            if l % R == 0:
                sa.select_pages(g, qs[l], summs[l], pt, sl, case.budget, case.sink,
                                case.window, ws, sel=sel, sel_count=cnt, k_cache=ks[l],
                                n_tail_refresh=1, sel_phys=phys)
            sa.attend_selected(g, qs[l], ks[l], vs[l], pt, sl, sel, cnt, case.scale, ws,
                               out=outs[l], lse=lses[l], sel_phys=phys)

    def step(with_events):
        for l in range(L_layers):
            if with_events:
                ev[l][0].record()
            sa.select_pages(g, qs[l], summs[l], pt, sl, case.budget, case.sink, case.window, ws,
                            sel=sel, sel_count=cnt, k_cache=ks[l], n_tail_refresh=1,
                            sel_phys=phys)
            if with_events:
                ev[l][1].record()
            sa.attend_selected(g, qs[l], ks[l], vs[l], pt, sl, sel, cnt, case.scale, ws,
                               out=outs[l], lse=lses[l], sel_phys=phys)
            if with_events:
                ev[l][2].record()

    # one eager step: correctness of the launch config, selection counts for the bytes
    step_fused()
    assert ws.status() == sa.SA_OK
    sel_count = cnt.cpu().numpy()
    sel_b, att_b, upd_b = layer_bytes(case.geom, case.seq_lens, sel_count, P, F8)
    n_sel_layers = (L_layers + R - 1) // R
    step_bytes = L_layers * att_b + n_sel_layers * (sel_b + upd_b)

    # the dominant kernel alone (page scoring of every layer), an event pair per launch
    ev_sc = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
             for _ in range(L_layers)]
    scores_buf = torch.empty((g.B, g.Hkv, g.max_pages), dtype=torch.float32, device=dev)

    def score_only():
        for l in range(L_layers):
            ev_sc[l][0].record()
            if F8:
                sa.page_scores_fp8(g, qs[l], summs[l], pt, sl, ws, scores=scores_buf)
            else:
                sa.page_scores(g, qs[l], summs[l], pt, sl, ws, scores=scores_buf)
            ev_sc[l][1].record()

    # capture: the step without events (headline), the step with per-phase events, and
    # the scoring launches with per-launch events
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    graph_ev = torch.cuda.CUDAGraph()
    graph_sc = torch.cuda.CUDAGraph()
    # (fp8 summaries have no separate selection call: no per-phase pass)
    with torch.cuda.stream(stream):
        if not F8:
            step(True)                  # warm the stream before capture
        step_fused()
        score_only()
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            step_fused()
        if not F8:
            with torch.cuda.graph(graph_ev, stream=stream):
                step(True)
        with torch.cuda.graph(graph_sc, stream=stream):
            score_only()
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    t0e = torch.cuda.Event(enable_timing=True)
    t1e = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t0e.record(stream)
        for _ in range(args.steps):
            graph.replay()
        t1e.record(stream)
    torch.cuda.synchronize()
    total_ms = t0e.elapsed_time(t1e)
    clk = clocks.stop()
    total_ms = max_over_ranks(total_ms, dist, dev)
    ms_per_step = total_ms / args.steps
    units_per_step = g.B * g.Hq * L_layers
    value = whole_job_rate(units_per_step, world, ms_per_step)
    step_gbs = step_bytes / (ms_per_step * 1e-3) / 1e9

    # ---- per-phase durations (events on the launching stream), averaged over replays
    sel_ms = np.zeros(L_layers)
    att_ms = np.zeros(L_layers)
    n_ev = max(3, args.steps // 2)
    sc_ms = np.zeros(L_layers)
    with torch.cuda.stream(stream):
        for _ in range(0 if F8 else n_ev):
            graph_ev.replay()
            torch.cuda.synchronize()
            for l in range(L_layers):
                sel_ms[l] += ev[l][0].elapsed_time(ev[l][1]) / n_ev
                att_ms[l] += ev[l][1].elapsed_time(ev[l][2]) / n_ev
        for _ in range(n_ev):
            graph_sc.replay()
            torch.cuda.synchronize()
            for l in range(L_layers):
                sc_ms[l] += ev_sc[l][0].elapsed_time(ev_sc[l][1]) / n_ev

    # ---- e2e through the public API with host buffers: q H2D + out/lse D2H every step
    q_host = [torch.empty(qs[l].shape, dtype=torch.int16).pin_memory() for l in range(L_layers)]
    for l in range(L_layers):
        q_host[l].copy_(qs[l].cpu())
    o_host = [torch.empty(outs[l].shape, dtype=torch.float32).pin_memory() for l in range(L_layers)]
    l_host = [torch.empty(lses[l].shape, dtype=torch.float32).pin_memory() for l in range(L_layers)]
    e2e_steps = max(3, args.steps // 2)
    with torch.cuda.stream(stream):
        for it in range(e2e_steps + 2):
            if it == 2:
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            for l in range(L_layers):
                qs[l].copy_(q_host[l], non_blocking=True)
            graph.replay()
            for l in range(L_layers):
                o_host[l].copy_(outs[l], non_blocking=True)
                l_host[l].copy_(lses[l], non_blocking=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    assert ws.status() == sa.SA_OK
    h2d = sum(int(x.numel()) * 2 for x in q_host)
    d2h = sum(int(x.numel()) * 4 for x in o_host) + sum(int(x.numel()) * 4 for x in l_host)

    if rank != 0:
        return 0
    att_mean = None if F8 else float(att_ms.mean())
    sel_mean = None if F8 else float(sel_ms.mean())
    sc_mean = float(sc_ms.mean())
    # page scoring: summaries + page-table entries + queries of one layer per launch
    dom_kernel = "score_mla_kernel" if g.v_aliases_k else (
        "score_stream_kernel<fp8>" if F8 else "score_stream_kernel")
    dom_bytes, dom_ms = sel_b, sc_mean
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    cpu_v, cpu_done, cpu_t, cpu_cores = (None, 0, 0.0, 0)
    cpu1 = (None, 0, 0.0)
    if world == 1:
        cpu_v, cpu_done, cpu_t, cpu_cores = oracle_sample_mt(case, args.cpu_seconds, R, F8)
        cpu1 = oracle_sample(case, args.cpu_seconds / 2, R, F8)
    extras = {}
    if world == 1 and args.extras and not g.v_aliases_k and R == 1 and not F8:
        # the same step as one persistent launch per layer (sa_sparse_decode_fused), timed
        # the headline's way on the headline's pools
        def step_single():
            for l in range(L_layers):
                sa.sparse_decode_fused(g, qs[l], ks[l], vs[l], summs[l], pt, sl, case.budget,
                                       case.sink, case.window, case.scale, ws, out=outs[l],
                                       lse=lses[l], sel_out=sel, sel_count_out=cnt,
                                       n_tail_refresh=1)
        try:
            with torch.cuda.stream(stream):
                step_single()
            torch.cuda.synchronize()
            graph_f = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_f, stream=stream):
                step_single()
            with torch.cuda.stream(stream):
                for _ in range(args.warmup):
                    graph_f.replay()
                torch.cuda.synchronize()
                f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                f0.record(stream)
                for _ in range(args.steps):
                    graph_f.replay()
                f1.record(stream)
            torch.cuda.synchronize()
            assert ws.status() == sa.SA_OK
            extras["single_launch_us_per_layer"] = (f0.elapsed_time(f1) * 1e3 /
                                                    (args.steps * L_layers))
            del graph_f
        except sa.SaError:
            extras["single_launch_us_per_layer"] = None
    if world == 1 and args.extras and args.workload == "llama32k" and R == 1 and not F8:
        # free the headline's pools first: the other configurations need the room
        del ks, vs, qs, summs, k0, v0, graph, graph_ev, graph_sc
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        for name in ("llama128k", "ragged", "mla"):
            extras.update(extra_decode(name, args, dev, hbm_peak))
    # GQA: score, select (+ tail refresh), attention, merge; latent: tail refresh, query
    # sign split, tensor-core score, select, tensor-core attention, merge
    # select half of one layer-call (the newest pages' refresh runs inside the scorer)
    launches_select = 4 if g.v_aliases_k else 2
    launches_attend = 2                           # attention + merge
    launches_per_step = n_sel_layers * launches_select + L_layers * launches_attend
    line = {
        "metric": "sparse-decode seq*heads/s",
        "value": value,
        "unit": "seq*heads/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            **workload_config(case, args, L_layers),
            "l2": "inputs larger than L2: %d distinct layer pools, %.2f GB touched per step"
                  % (L_layers, step_bytes / 1e9),
            "parallelism": "replicas (batch split), no collective" if world > 1 else "1 GPU",
            "step_hbm_gbs": step_gbs,
            "step_frac_of_hbm_peak": step_gbs / hbm_peak,
            "us_per_layer": ms_per_step * 1e3 / L_layers,
            "select_pages_us_alone": None if sel_mean is None else sel_mean * 1e3,
            "attend_selected_us_alone": None if att_mean is None else att_mean * 1e3,
            "page_scores_us_alone": sc_mean * 1e3,
            "summaries_us_alone": summ_ms * 1e3,
            "summaries_gbs_alone": summ_bytes / (summ_ms * 1e-3) / 1e9,
            "algorithmic_bytes_per_layer": step_bytes / L_layers,
            **mla_flops(case, sel_count, sc_mean, att_mean),
            **extras,
        },
        "roofline": {
            "kernel": dom_kernel,
            "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
            "frac": achieved / hbm_peak, "peak_kind": peak_kind + " (burst copy)",
            "bytes_per_launch": dom_bytes,
            "traffic": recorded_traffic(dom_kernel, args.workload),
        },
        "cpu_baseline": None if cpu_v is None else {
            "value": cpu_v, "unit": "seq*heads/s", "cores": cpu_cores, "kind": "oracle",
            "sample": "%d (sequence, layer) decode calls of layer 0 (score+select%s, attend; "
                      "all %d query heads) on %d host threads (independent sequences), "
                      "%.1f s wall" % (cpu_done, "" if R == 1 else " every %d layers" % R,
                                       g.Hq, cpu_cores, cpu_t),
            "single_thread_value": cpu1[0],
            "single_thread_sample": "%d calls, %.1f s on one thread" % (cpu1[1], cpu1[2])},
        "e2e": {"value": whole_job_rate(units_per_step, world, e2e_ms), "unit": "seq*heads/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    print(json.dumps(line, default=_json_default), flush=True)
    return 0


def extra_decode(name, args, dev, hbm_peak, layers=8, steps=10, warmup=3):
    """One more decode configuration timed the headline's way (a CUDA graph of `layers`
    sa_sparse_decode calls over distinct layer pools, inputs resident, CUDA events), for
    the line's config: microseconds per layer-call and the fraction of HBM peak at the
    algorithmic bytes; the latent geometry adds its tensor-core rate."""
    import torch
    import paged_kv_cache_sa_b200 as sa
    from paged_kv_cache_sa_b200 import Geometry

    case = synth.decode_case(name, seed=rank_seed(name, 0, args.seed))
    g = Geometry.of(case.geom)
    P = g.P
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16
                                                          else a)).to(dev)
    k0 = t(case.k_cache)
    v0 = t(case.v_cache) if case.v_cache is not None else None
    pt, sl = t(case.page_table), t(case.seq_lens)
    rng = np.random.default_rng(4321)
    stride = max(1, g.n_pool // layers)
    ks, vs, qs, summs = [], [], [], []
    for l in range(layers):
        ks.append(k0 if l == 0 else torch.roll(k0, shifts=l * stride, dims=0))
        vs.append(None if v0 is None else (v0 if l == 0 else torch.roll(v0, shifts=l * stride, dims=0)))
        qn = case.q if l == 0 else synth.f32_to_bf16(rng.standard_normal(case.q.shape).astype(np.float32))
        qs.append(t(qn))
        summs.append(torch.empty((g.n_pool, g.Hkv, 2, g.Dk), dtype=torch.int16, device=dev))
        sa.page_summaries(g, ks[l], pt, sl, summs[l])
    K = case.budget // P
    ws = sa.Workspace.for_decode(g, case.budget)
    sel = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device=dev)
    cnt = torch.empty((g.B, g.Hkv), dtype=torch.int32, device=dev)
    out = torch.empty((g.B, g.Hq, g.Dv), dtype=torch.float32, device=dev)
    lse = torch.empty((g.B, g.Hq), dtype=torch.float32, device=dev)

    def run():
        for l in range(layers):
            sa.sparse_decode(g, qs[l], ks[l], vs[l], summs[l], pt, sl, case.budget, case.sink,
                             case.window, case.scale, ws, out=out, lse=lse, sel_out=sel,
                             sel_count_out=cnt, n_tail_refresh=1)

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize()
    assert ws.status() == sa.SA_OK
    sel_count = cnt.cpu().numpy()
    sel_b, att_b, upd_b = layer_bytes(case.geom, case.seq_lens, sel_count, P)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        run()
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    assert ws.status() == sa.SA_OK
    us = e0.elapsed_time(e1) * 1e3 / (steps * layers)
    layer_b = sel_b + att_b + upd_b
    res = {
        name + "_us_per_layer": us,
        name + "_algorithmic_bytes_per_layer": layer_b,
        name + "_frac_of_hbm_peak": layer_b / (us * 1e-6) / 1e9 / hbm_peak,
        name + "_layers_timed": layers,
    }
    if g.v_aliases_k:
        fl = mla_flops(case, sel_count, 1.0, 1.0)
        tot = (fl["score_gflop_per_layer"] + fl["attend_gflop_per_layer"]) * 1e9
        res[name + "_tensor_tflops"] = tot / (us * 1e-6) / 1e12
    del graph, ks, vs, qs, summs, k0, v0
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def mla_flops(case, sel_count, score_ms, attend_ms):
    """Latent geometry: tensor-core work per layer (scores as a GEMM over 2*Dk, Q.K^T
    and P.V over the selected tokens) and its rate in the timed-alone phases."""
    g = case.geom
    if not g.v_aliases_k:
        return {}
    P = g.P
    nb = (case.seq_lens.astype(np.int64) + P - 1) // P
    score_f = 2.0 * g.Hq * 2 * g.Dk * float(nb.sum())
    tok = 0
    for b in range(g.B):
        L = int(case.seq_lens[b])
        last = L - (int(nb[b]) - 1) * P if nb[b] else 0
        c = int(sel_count[b, 0])
        tok += c * P - (P - last if c else 0)
    att_f = 2.0 * g.Hq * (g.Dk + g.Dv) * tok
    return {"score_gflop_per_layer": score_f / 1e9, "attend_gflop_per_layer": att_f / 1e9,
            "score_tflops_alone": score_f / (score_ms * 1e-3) / 1e12,
            "attend_tflops_alone": att_f / (attend_ms * 1e-3) / 1e12}


# ------------------------------------------------------------------------------------
# prune workload: compaction of every session, then one decode over the compacted cache
# ------------------------------------------------------------------------------------

def prune_bytes(case, keep):
    """Algorithmic bytes of one compaction: kept tokens read and written (K and V, every
    KV head), the keep-mask, the new pages' summaries and tables."""
    g = case.geom
    kept = 0
    pages = 0
    for b in range(g.B):
        L = int(case.seq_lens[b])
        k = int(keep[b, :L].sum())
        kept += k
        pages += (k + g.P - 1) // g.P
    row = g.Hkv * (g.Dk + (0 if g.v_aliases_k else g.Dv)) * 2
    mask = int(case.seq_lens.sum())
    return 2 * kept * row + mask + pages * g.Hkv * 2 * g.Dk * 2 + g.B * g.max_pages * 4, kept


def oracle_prune_sample(pc, seconds):
    """Time the CPU oracle's compaction session by session until ~`seconds` elapsed."""
    import oracle
    d = pc.decode
    g = d.geom
    done, t_total, b = 0, 0.0, 0
    fp_off = 0
    while t_total < seconds and done < g.B:
        sub = synth.Geometry(1, g.Hq, g.Hkv, g.Dk, g.Dv, g.P, g.max_pages, g.n_pool, g.v_aliases_k)
        L = int(d.seq_lens[b])
        need = (int(pc.keep[b, :L].sum()) + g.P - 1) // g.P
        t0 = time.perf_counter()
        oracle.prune_compact(sub, d.k_cache, d.v_cache, d.page_table[b:b + 1], d.seq_lens[b:b + 1],
                             pc.keep[b:b + 1], pc.free_pages[fp_off:fp_off + need])
        t_total += time.perf_counter() - t0
        fp_off += need
        done += 1
        b += 1
    return done / t_total, done, t_total


def run_prune(args, rank, world, dist):
    import torch
    import paged_kv_cache_sa_b200 as sa
    from paged_kv_cache_sa_b200 import Geometry

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    hbm_peak, _, peak_kind = peaks()
    pc = synth.prune_case("prune", seed=rank_seed("prune", rank, args.seed))
    d = pc.decode
    g = Geometry.of(d.geom)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16
                                                          else a)).to(dev)
    k, v = t(d.k_cache), t(d.v_cache)
    pt, sl, keep, fp = t(d.page_table), t(d.seq_lens), t(pc.keep), t(pc.free_pages)
    q = t(d.q)
    summ = torch.zeros((g.n_pool, g.Hkv, 2, g.Dk), dtype=torch.int16, device=dev)
    wsp = sa.Workspace.for_prune(g)
    wsd = sa.Workspace.for_decode(g, d.budget)
    width = g.max_pages * g.P
    npt = torch.empty((g.B, g.max_pages), dtype=torch.int32, device=dev)
    nsl = torch.empty((g.B,), dtype=torch.int32, device=dev)
    pos = torch.empty((g.B, width), dtype=torch.int32, device=dev)
    ll = torch.empty((g.B,), dtype=torch.int32, device=dev)
    out = torch.empty((g.B, g.Hq, g.Dv), dtype=torch.float32, device=dev)
    lse = torch.empty((g.B, g.Hq), dtype=torch.float32, device=dev)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]

    def step(with_events):
        # compaction into the fresh pages (the old pages stay readable: repeating the
        # step rewrites the same bytes), then one decode over the compacted cache
        if with_events:
            ev[0].record()
        sa.prune_compact(g, k, v, pt, sl, keep, fp, k, v, summ, wsp, new_page_table=npt,
                         new_seq_lens=nsl, pos_map=pos, logical_len=ll)
        if with_events:
            ev[1].record()
        sa.sparse_decode(g, q, k, v, summ, npt, nsl, d.budget, d.sink, d.window, d.scale, wsd,
                         out=out, lse=lse)
        if with_events:
            ev[2].record()

    step(False)
    torch.cuda.synchronize()
    assert wsp.status() == sa.SA_OK and wsd.status() == sa.SA_OK
    pbytes, kept = prune_bytes(d, pc.keep)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph, graph_ev = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        step(True)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            step(False)
        with torch.cuda.graph(graph_ev, stream=stream):
            step(True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0e.record(stream)
        for _ in range(args.steps):
            graph.replay()
        t1e.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms_per_step = max_over_ranks(t0e.elapsed_time(t1e), dist, dev) / args.steps
    prune_ms = dec_ms = 0.0
    n_ev = max(3, args.steps // 2)
    with torch.cuda.stream(stream):
        for _ in range(n_ev):
            graph_ev.replay()
            torch.cuda.synchronize()
            prune_ms += ev[0].elapsed_time(ev[1]) / n_ev
            dec_ms += ev[1].elapsed_time(ev[2]) / n_ev
    assert wsp.status() == sa.SA_OK and wsd.status() == sa.SA_OK
    # e2e: the query in and the outputs out every step, through pinned host buffers
    q_host = torch.empty(q.shape, dtype=torch.int16).pin_memory()
    q_host.copy_(q.cpu())
    o_host = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    l_host = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    e2e_steps = max(3, args.steps // 2)
    with torch.cuda.stream(stream):
        for it in range(e2e_steps + 2):
            if it == 2:
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            q.copy_(q_host, non_blocking=True)
            graph.replay()
            o_host.copy_(out, non_blocking=True)
            l_host.copy_(lse, non_blocking=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dist, dev)
    if rank != 0:
        return 0
    units = g.B * g.Hq
    achieved = pbytes / (prune_ms * 1e-3) / 1e9
    cpu_v = cpu_done = cpu_t = None
    if world == 1:
        cpu_v, cpu_done, cpu_t = oracle_prune_sample(pc, args.cpu_seconds)
    line = {
        "metric": "sparse-decode seq*heads/s", "value": whole_job_rate(units, world, ms_per_step),
        "unit": "seq*heads/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": "prune", "sessions": g.B, "q_heads": g.Hq, "kv_heads": g.Hkv,
            "head_dim": g.Dk, "page": g.P, "kept_tokens": kept,
            "tokens_before": int(d.seq_lens.sum()), "budget_tokens": d.budget,
            "step": "sa_prune_compact of every session + one sa_sparse_decode over the "
                    "compacted cache",
            "l2": "inputs larger than L2: %.2f GB of K/V pool" % (
                (k.numel() + v.numel()) * 2 / 1e9),
            "prune_us_alone": prune_ms * 1e3, "decode_us_alone": dec_ms * 1e3,
            "prune_algorithmic_bytes": pbytes,
        },
        "roofline": {"kernel": "sa_prune_compact (count, plan, position, copy kernels)",
                     "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_kind": peak_kind + " (burst copy)",
                     "bytes_per_launch": pbytes, "traffic": None},
        "cpu_baseline": None if cpu_v is None else {
            "value": cpu_v, "unit": "sessions compacted/s", "cores": 1, "kind": "oracle",
            "sample": "%d of %d sessions compacted by the oracle, %.1f s single-threaded" % (
                cpu_done, g.B, cpu_t)},
        "e2e": {"value": whole_job_rate(units, world, e2e_ms), "unit": "seq*heads/s",
                "h2d_bytes_per_step": int(q.numel()) * 2,
                "d2h_bytes_per_step": int(out.numel() + lse.numel()) * 4},
        "gpu_launches": 8 * args.steps,  # prune: 4 kernels; decode: 4 kernels
        "clocks": clk,
    }
    print(json.dumps(line, default=_json_default), flush=True)
    return 0


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, or None when
    there is none for this workload or the kernel's source changed since it was taken.
    The source is hashed without its SA_TRACE_POINT lines, which expand to nothing
    outside the traced build."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[kernel]
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("workload") != workload:
        return None
    src = os.path.join(ROOT, "paged_kv_cache_sa_b200", "csrc", rec["source"])
    try:
        text = open(src, "rb").read().decode()
        text = "".join(l for l in text.splitlines(True) if "SA_TRACE_POINT" not in l)
        sha = hashlib.sha256(text.encode()).hexdigest()
    except OSError:
        return None
    return rec["dram_bytes_per_launch"] if sha == rec["source_sha256"] else None


def main():
    args = parse()
    if args.select_every < 1:
        raise SystemExit("--select-every must be >= 1")
    if args.layers is None:
        args.layers = N_LAYERS if args.workload == "llama32k" else 8
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        if args.impl == "native":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        # the native arm's ranks time GPUs (NCCL); the oracle arm runs on host cores (gloo)
        tdist.init_process_group("nccl" if args.impl == "native" else "gloo",
                                 timeout=datetime.timedelta(seconds=300))
        dist = tdist
    try:
        if args.impl == "reference":
            rc = run_reference(args, rank, world)
        elif args.workload == "prune":
            rc = run_prune(args, rank, world, dist)
        else:
            rc = run_native(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
