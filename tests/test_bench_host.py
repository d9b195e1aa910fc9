"""Host logic of bench.py (CPU): committed traffic figures are used only while
the sources they were measured on are unchanged, and scale by algorithmic bytes."""
import json

import bench


def test_decode_traffic_follows_source_hash(tmp_path, monkeypatch):
    path = tmp_path / "decode_traffic.json"
    monkeypatch.setattr(bench, "DECODE_TRAFFIC_PATH", str(path))
    good = bench.kernel_source_hash(("decode.cu", "sm100_ptx.cuh", "g3_internal.h"))
    path.write_text(json.dumps({"bytes_per_algorithmic_byte": 1.25, "source_hash": good}))
    assert bench.decode_traffic_per_launch(1000.0) == 1250.0
    path.write_text(json.dumps({"bytes_per_algorithmic_byte": 1.25, "source_hash": "0" * 16}))
    assert bench.decode_traffic_per_launch(1000.0) is None
    path.write_text("not json")
    assert bench.decode_traffic_per_launch(1000.0) is None


def test_source_hash_depends_on_the_files():
    a = bench.kernel_source_hash(("prefill.cu",))
    b = bench.kernel_source_hash(("prefill.cu", "g3_internal.h"))
    assert a != b and len(a) == 16
    assert a == bench.kernel_source_hash(("prefill.cu",))


def test_weak_scaling_rate_counts_every_rank():
    # 2 ranks x 3 steps of 10 units in 6 ms (the slowest rank) = 10,000 units/s
    assert bench.weak_scaling_rate(10.0, 3, 2, 6.0) == 10.0 * 3 * 2 / 6e-3


def test_trace_sampling_counts():
    # The trace rides on steps 0, TRACE_EVERY, 2*TRACE_EVERY, ... of the timed loop.
    E = bench.TRACE_EVERY
    assert bench.n_traced(1) == 1
    assert bench.n_traced(E) == 1
    assert bench.n_traced(E + 1) == 2
    assert bench.n_traced(20) == len(range(0, 20, E))
    # 12 launches per step on the traced steps scale to every timed step.
    steps = 20
    trace = {"prefill_prologue": (6 * bench.n_traced(steps), 1.0),
             "prefill_attention": (6 * bench.n_traced(steps), 9.0)}
    assert bench.launches_in_timed_region(trace, steps) == 12 * steps
    # plus the untraced device-error reset kernel of each of the six prefill calls
    assert bench.launches_in_timed_region(trace, steps, untraced_per_step=6) == 18 * steps


def test_long_block_spans_are_the_workloads():
    # the mixed block: 8 images of 256 tokens per sequence, sorted, disjoint and
    # inside the sequence; the same set serves every layer of the block
    import numpy as np
    import inputs
    cfg = inputs.MIXED_32K
    sp = bench.long_block_spans(cfg).numpy()
    assert sp.shape == (cfg.B, cfg.n_spans, 2)
    assert ((sp[:, :, 1] - sp[:, :, 0]) == 256).all()
    assert (sp[:, 1:, 0] >= sp[:, :-1, 1]).all() and sp.min() >= 0 and sp.max() <= cfg.S
    assert np.array_equal(sp, bench.long_block_spans(cfg).numpy())
    assert bench.long_block_spans(inputs.LONG_128K) is None


def test_fractions_of_measured_and_nominal_peaks():
    f = bench.fractions(750.0, 1618.8, bench.NOMINAL["bf16_tflops"])
    assert abs(f["of_measured"] - 750.0 / 1618.8) < 1e-12
    assert abs(f["of_nominal"] - 750.0 / 2250.0) < 1e-12
    assert bench.fractions(1.0, 0.0, 2.0)["of_measured"] is None
