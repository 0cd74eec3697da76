"""CPU checks of bench.py's oracle legs (cpu_baseline and --impl reference):
the operands assembled once are those the oracle's stream attention uses, the
timed call computes exactly its result on the sampled rows, the sample grows
to the time target, and the baseline entry carries the fields the JSON line
needs."""
import importlib.util
import os
import sys

import numpy as np

import oracle
from causal_attention_rtr_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    try:
        sys.argv = ["bench.py"]
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_oracle_rows_equal_stream_attention():
    bench = _bench()
    w = synth.TINY_F32
    x = synth.stream_layer_inputs(w)
    ops = bench.oracle_operands(w, x)
    rows = np.array([0, 3, 7, w.chunk_frames * w.k - 1])
    got = bench.oracle_rows(w, ops, rows)
    want = bench.oracle_cache_for(w, x).stream_attention(x.q, x.k_cur, x.v_cur, w.chunk_frames, rows=rows)
    assert np.array_equal(got, want)
    assert np.array_equal(bench.oracle_rows(w, ops, rows, nthreads=1), want)


def test_time_oracle_and_baseline_entry():
    bench = _bench()
    w = synth.TINY_F32
    x = synth.stream_layer_inputs(w)
    ops = bench.oracle_operands(w, x)
    flops, dt, rows = bench.time_oracle(w, ops, 0.001)
    assert dt > 0 and len(rows) >= 2 and flops == bench.oracle_sample_flops(w, rows)
    entry = bench.cpu_baseline_entry(flops, dt, rows, w)
    assert entry["kind"] == "oracle" and entry["unit"] == "TFLOP/s" and entry["value"] > 0
    assert entry["cores"] == oracle.max_threads() >= 1
    assert str(len(rows)) in entry["sample"]


def test_oracle_sample_flops_counts_visible_pairs():
    """4 d flops per visible (query, key) pair per head: a chunk row of frame
    c sees the cached frames and chunk frames 0..c."""
    bench = _bench()
    w = synth.WAN13_LAYER
    cached = (w.ref_frames + w.window_frames) * w.k
    rows = np.array([0, w.k, 2 * w.k + 5])
    want = sum(4.0 * w.head_dim * w.heads * (cached + (c + 1) * w.k) for c in (0, 1, 2))
    assert bench.oracle_sample_flops(w, rows) == want
