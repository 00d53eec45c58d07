"""The phase-timeline build (lib/libsa_trace.so, include/sa_trace.h) against libsa.so.

- It computes bitwise the same selection, output and log-sum-exp as libsa.so.
- Its %globaltimer stamps respect the order the kernels' dependency waits promise: the
  selection sees the scores only after every scoring CTA's last stamp, the attention sees
  the selection only after every selection CTA has written its list, and the merge sees
  the attention only after every attention warp has finished its range.
"""

import ctypes
import os

import numpy as np
import pytest

import synth
from parity import DevCase

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import paged_kv_cache_sa_b200 as sa  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SLACK_NS = 64  # timer granularity


def _traced_lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_sa_build", os.path.join(ROOT, "paged_kv_cache_sa_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    lib = sa._load(b.build(trace=True))
    lib.sa_trace_set.argtypes = [ctypes.c_void_p]
    lib.sa_trace_set.restype = ctypes.c_int
    return lib


def _decode(dc, case, ws):
    g = dc.g
    K = case.budget // g.P
    sel = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device="cuda")
    cnt = torch.empty((g.B, g.Hkv), dtype=torch.int32, device="cuda")
    out, lse = sa.sparse_decode(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, case.budget,
                                case.sink, case.window, case.scale, ws, sel_out=sel,
                                sel_count_out=cnt, n_tail_refresh=1)
    assert ws.status() == sa.SA_OK
    return [t.cpu().numpy() for t in (sel, cnt, out, lse)]


def test_traced_build_same_results_and_ordered_stamps():
    case = synth.decode_case("llama32k", B=4, L=(16384, 32768), seed=17)
    dc = DevCase(case)
    g = dc.g
    sa.page_summaries(g, dc.k, dc.pt, dc.sl, dc.summ)
    ws = sa.Workspace.for_decode(g, case.budget)
    ref = _decode(dc, case, ws)
    lib = _traced_lib()
    plain = sa.lib
    buf = torch.zeros(5 * 1024 * 16, dtype=torch.int64, device="cuda")
    try:
        sa.lib = lib
        assert lib.sa_trace_set(ctypes.c_void_p(buf.data_ptr())) == sa.SA_OK
        got = _decode(dc, case, ws)
        torch.cuda.synchronize()
    finally:
        lib.sa_trace_set(None)
        sa.lib = plain
    for a, b in zip(ref, got):
        assert np.array_equal(a, b)
    t = buf.view(5, 1024, 16).cpu().numpy().astype(np.int64)

    def stamps(kid, evs):
        v = t[kid][:, evs]
        return v[v > 0]

    score_all = stamps(0, list(range(5)))
    sel_visible = stamps(1, [0])
    sel_written = stamps(1, [3])
    att_visible = stamps(2, [2])
    att_done = stamps(2, list(range(5, 13)))
    merge_visible = stamps(3, [1])
    n_pairs = g.B * g.Hkv
    assert sel_visible.size == n_pairs and sel_written.size == n_pairs
    assert score_all.size > 0 and att_visible.size > 0 and att_done.size > 0
    assert merge_visible.size > 0
    # per scoring CTA: entry <= dependency wait passed <= slice tables ready
    rows = t[0][:, :3]
    rows = rows[(rows > 0).all(axis=1)]
    assert rows.shape[0] > 0
    assert (np.diff(rows, axis=1) >= 0).all()
    # every dependency wait passes after everything the previous grid stamped
    assert score_all.max() <= sel_visible.min() + SLACK_NS
    assert sel_written.max() <= att_visible.min() + SLACK_NS
    assert att_done.max() <= merge_visible.min() + SLACK_NS
