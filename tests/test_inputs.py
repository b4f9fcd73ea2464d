"""The seeded generators: determinism and the ignore/label recipe per workload."""
import numpy as np

import flce_inputs as fi


def test_tiny_is_deterministic_and_quantised():
    a = fi.make_inputs("tiny", keep_raw=True)
    b = fi.make_inputs("tiny", threads=1)
    assert np.array_equal(a.hidden_bits, b.hidden_bits)
    assert np.array_equal(a.weight_bits, b.weight_bits)
    assert np.array_equal(a.labels, b.labels)
    # quantisation error is at most half a bf16 ulp: 2^-8 relative (8-bit significand)
    rel = np.abs(a.hidden - a.hidden_raw) / np.abs(a.hidden_raw)
    assert rel.max() <= 2.0 ** -8
    assert a.hidden_bits.dtype == np.uint16 and a.hidden.dtype == np.float32


def test_label_recipes():
    for name, w in fi.WORKLOADS.items():  # includes the profiling-size problem
        y = fi._draw_labels(w)
        assert y.shape == (w.N,) and y.dtype == np.int64
        valid = y != fi.IGNORE_INDEX
        assert np.all((y[valid] >= 0) & (y[valid] < w.V))
        if w.ignore_rule == "count":
            assert (~valid).sum() == w.ignore_count
        elif w.ignore_rule == "tail":
            assert (~valid).sum() == w.ignore_count
            assert np.all(~valid[-w.ignore_count:]) and np.all(valid[:-w.ignore_count])
        else:
            mb = w.N // w.microbatches
            for k in range(w.microbatches):
                nk = (~valid[k * mb:(k + 1) * mb]).sum()
                assert nk == (mb if k == w.empty_microbatch else w.ignore_count)


def test_zipf_labels_are_heavy_headed():
    y = fi._draw_labels(fi.WORKLOADS["v131k_zipf"])
    y = y[y >= 0]
    # Zipf(1.1): token 0 is the most frequent and the head holds a large share
    counts = np.bincount(y, minlength=10)
    assert counts[0] == counts.max()
    assert (y < 100).mean() > 0.3


def test_percentages_of_the_workloads():
    w = fi.WORKLOADS
    assert w["tiny"].ignore_count == 64 // 4
    assert w["v32k_mean"].ignore_count == int(0.10 * 4096)
    assert w["v131k_zipf"].ignore_count == int(0.05 * 16384)
    assert w["v256k_softcap"].ignore_count == round(0.2 * 8192)
    assert w["microbatch"].ignore_count == int(0.30 * 4096)
