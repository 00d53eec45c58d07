"""Phase timeline of one decode call on the GPU, from the traced build of the library.

    python paged_kv_cache_sa_b200/timeline.py [--workload llama32k] [--fused]

Builds lib/libsa_trace.so (the same sources with -DSA_TRACE, include/sa_trace.h), makes
three layer pools of the seeded workload (so the timed call's inputs are not in L2),
warms up, then records one sa_sparse_decode (or sa_sparse_decode_fused) call and prints,
for each trace point, the median, min and max over the CTAs that reached it, in µs from
the first scoring CTA's start.  The trace stores add a few stores per CTA; the untraced
per-call time is printed beside it.
"""

from __future__ import annotations

import argparse
import ctypes
import os
import sys

import numpy as np

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# (kernel, event) -> name
EVENTS = {
    0: ["entry", "dependency wait passed", "slice tables ready", "first stage (consumer 0)",
        "consumer 0 done"],
    1: ["scores visible", "keys and range", "threshold", "list written",
        "keys stored (thread 0)", "histogram built", "boundary bin found", "list counts"],
    2: ["entry", "lengths-only tables", "selection visible", "unit tables ready",
        "first unit (warp 0)"] + ["warp %d done" % w for w in range(8)] +
       ["unit loads landed"],
    3: ["entry", "attention visible"],
    4: ["phase 1 done", "phase 2 done", "barrier 2 passed", "phase 3 done",
        "barrier 3 passed"],
}
KERNELS = ["scoring", "selection", "attention", "merge", "single launch"]


def main():
    ap = argparse.ArgumentParser()
    # the grouped-query workloads: the latent geometry's kernels carry no trace points
    ap.add_argument("--workload", default="llama32k",
                    choices=["tiny", "llama32k", "llama128k", "ragged"])
    ap.add_argument("--fused", action="store_true", help="time sa_sparse_decode_fused")
    args = ap.parse_args()

    import importlib.util
    spec = importlib.util.spec_from_file_location("_sa_build", os.path.join(PKG, "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    path = b.build(trace=True)

    import torch
    import synth
    import paged_kv_cache_sa_b200 as sa
    lib = sa._load(path)
    lib.sa_trace_set.argtypes = [ctypes.c_void_p]
    lib.sa_trace_set.restype = ctypes.c_int
    sa.lib = lib

    case = synth.decode_case(args.workload)
    g = sa.Geometry.of(case.geom)
    dev = torch.device("cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(
        a.view(np.int16) if a.dtype == np.uint16 else a)).to(dev)
    k0, v0 = t(case.k_cache), t(case.v_cache)
    pt, sl = t(case.page_table), t(case.seq_lens)
    n = 3
    ks = [torch.roll(k0, shifts=l * g.n_pool // n, dims=0) for l in range(n)]
    vs = [torch.roll(v0, shifts=l * g.n_pool // n, dims=0) for l in range(n)]
    q = t(case.q)
    summs = []
    for l in range(n):
        s_ = torch.empty((g.n_pool, g.Hkv, 2, g.Dk), dtype=torch.int16, device=dev)
        sa.page_summaries(g, ks[l], pt, sl, s_)
        summs.append(s_)
    ws = sa.Workspace.for_decode(g, case.budget)
    out = torch.empty((g.B, g.Hq, g.Dv), dtype=torch.float32, device=dev)
    lse = torch.empty((g.B, g.Hq), dtype=torch.float32, device=dev)
    fn = sa.sparse_decode_fused if args.fused else sa.sparse_decode

    def call(l):
        fn(g, q, ks[l], vs[l], summs[l], pt, sl, case.budget, case.sink, case.window,
           case.scale, ws, out=out, lse=lse, n_tail_refresh=1)

    lib.sa_trace_set(None)
    for i in range(6):
        call(i % n)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(30):
        call(i % n)
    e1.record()
    torch.cuda.synchronize()
    print("%s, %s: %.2f us per call untraced (eager launches)" % (
        args.workload, "sa_sparse_decode_fused" if args.fused else "sa_sparse_decode",
        e0.elapsed_time(e1) / 30 * 1e3))
    buf = torch.zeros(5 * 1024 * 16, dtype=torch.int64, device=dev)
    lib.sa_trace_set(ctypes.c_void_p(buf.data_ptr()))
    call(1)
    call(2)
    torch.cuda.synchronize()
    buf.zero_()
    torch.cuda.synchronize()
    call(0)
    torch.cuda.synchronize()
    lib.sa_trace_set(None)
    assert ws.status() == sa.SA_OK
    a = buf.view(5, 1024, 16).cpu().numpy().astype(np.int64)
    start = a[0, :, 0][a[0, :, 0] > 0]
    if start.size == 0:
        raise SystemExit("no trace recorded")
    t0 = start.min()
    print("%-13s %-26s %5s %9s %9s %9s" % ("kernel", "point (by median)", "CTAs", "median",
                                         "min", "max"))
    for kid, names in EVENTS.items():
        rows = []
        for ev, name in enumerate(names):
            v = a[kid, :, ev]
            v = v[v > 0]
            if v.size:
                v = (v - t0) / 1e3
                rows.append((np.median(v), name, v))
        for med, name, v in sorted(rows, key=lambda r: r[0]):
            print("%-13s %-26s %5d %9.2f %9.2f %9.2f" % (
                KERNELS[kid], name, v.size, med, v.min(), v.max()))


if __name__ == "__main__":
    main()
