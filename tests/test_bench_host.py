"""Host-side pieces of bench.py, on CPU: the algorithmic byte count per layer-call (bf16
and fp8 summaries), the oracle's timed sample, and the lookup of the committed DRAM
traffic records."""

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def test_layer_bytes_by_summary_format():
    case = synth.decode_case("llama32k", B=2, seq_lens=[4096, 1000], seed=3)
    g = case.geom
    cnt = np.full((g.B, g.Hkv), case.budget // g.P, dtype=np.int32)
    cnt[1] = (1000 + g.P - 1) // g.P                      # short sequence: all its pages
    s16, a16, u16 = bench.layer_bytes(g, case.seq_lens, cnt, g.P)
    s8, a8, u8 = bench.layer_bytes(g, case.seq_lens, cnt, g.P, fp8=True)
    nb = (4096 + 15) // 16 + (1000 + 15) // 16
    other = nb * 4 + g.B * g.Hq * g.Dk * 2                 # page table + q
    assert s16 - other == nb * g.Hkv * 4 * g.Dk            # bf16 min/max rows
    assert s8 - other == nb * g.Hkv * (2 * g.Dk + 16)      # fp8 records
    assert a16 == a8                                       # attention reads bf16 K, V alike
    # K+V of the selected valid tokens: sequence 0 full pages, sequence 1 ends at 1000
    tok = g.Hkv * (128 * 16 + 1000)
    assert a16 == tok * 2 * g.Dk * 2 + g.B * g.Hq * g.Dk * 2 + g.B * g.Hq * (g.Dv * 4 + 4)
    assert u16 - u8 == g.B * g.Hkv * (4 * g.Dk - (2 * g.Dk + 16))


def test_oracle_sample_both_formats_and_reuse():
    case = synth.decode_case("tiny", B=2, seq_lens=[4096, 700], Hkv=1, Hq=4)
    for fp8 in (False, True):
        for r in (1, 3):
            v, done, t = bench.oracle_sample(case, 0.05, select_every=r, fp8=fp8)
            assert done >= 1 and t > 0 and v > 0


def test_recorded_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu record only while the kernel's source
    is the one measured; SA_TRACE_POINT lines (nothing outside the traced build) do not
    count as a change."""
    import hashlib
    import json
    src_dir = tmp_path / "paged_kv_cache_sa_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    body = "int a;\nint b;\n"
    sha = hashlib.sha256(body.encode()).hexdigest()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({
        "k": {"workload": "llama32k", "source": "x.cuh", "source_sha256": sha,
              "dram_bytes_per_launch": 1234}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    src = src_dir / "x.cuh"
    src.write_text(body)
    assert bench.recorded_traffic("k", "llama32k") == 1234
    assert bench.recorded_traffic("k", "llama128k") is None      # another workload
    assert bench.recorded_traffic("other", "llama32k") is None   # no record
    src.write_text("int a;\n  SA_TRACE_POINT(0, 1);  // stamp\nint b;\n")
    assert bench.recorded_traffic("k", "llama32k") == 1234
    src.write_text("int a;\nint c;\n")
    assert bench.recorded_traffic("k", "llama32k") is None       # the kernel changed


def test_reference_arm_config_matches_the_native_line():
    """The reference arm describes the workload with the native line's static keys: the
    same L2 and parallelism wording and the same algorithmic bytes (llama32k, 32 layers:
    134,841,344 B per layer-call, the figure the native bench prints from its measured
    selection counts)."""
    import argparse
    case = synth.decode_case("llama32k")
    args = argparse.Namespace(workload="llama32k", summaries="bf16", select_every=1)
    cnt = bench.selection_counts(case)
    assert cnt.shape == (case.geom.B, case.geom.Hkv)
    assert (cnt == case.budget // case.geom.P).all()
    sb = bench.step_bytes_of(case, args, 32, cnt)
    cfg = bench.run_config(case, args, 32, 1, sb)
    assert cfg["algorithmic_bytes_per_layer"] == 134841344
    assert cfg["l2"] == "inputs larger than L2: 32 distinct layer pools, 4.31 GB touched per step"
    assert cfg["parallelism"] == "1 GPU"
    assert bench.run_config(case, args, 32, 2, sb)["parallelism"].startswith("replicas")
    # short sequences select all their pages
    short = synth.decode_case("tiny", B=2, seq_lens=[4096, 100], Hkv=1, Hq=4)
    assert bench.selection_counts(short).tolist() == [[short.budget // 16], [7]]
