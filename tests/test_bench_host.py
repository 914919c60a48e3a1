"""Host-side pieces of bench.py that run without a GPU: the CPU baseline of a
stack (the oracle's forward of one layer, extrapolated over the layers) and
the source sections whose hash ties the reported DRAM traffic to the capture
it came from."""
import os
import sys

import pytest

import synthetic as syn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_stack_decode_cpu_baseline_is_the_layer_rate_over_the_layers():
    w = syn.Workload("tiny-stack", T=8, D=64, F=128, V=100, layers=4, dtype="bf16", w_std=0.05,
                     e_std=0.05, x_std=1.0, dy_std=1.0, table="device", cache_frac=0.0, group=1,
                     training=False)
    r = bench.cpu_baseline_stack_decode(w, seconds=0.2)
    assert r["kind"] == "oracle" and r["unit"] == "tokens/s" and r["cores"] >= 1
    assert r["value"] > 0
    assert "extrapolated to 4 layers" in r["sample"]


def test_captured_traffic_sources_exist_and_sections_are_found():
    for name, c in bench.CAPTURED_TRAFFIC.items():
        assert os.path.exists(os.path.join(ROOT, c["profile"])), c["profile"]
        for f, first, end in c["sources"]:
            text = open(os.path.join(ROOT, f)).read()
            if first is not None:
                i = text.find(first)
                assert i >= 0, (f, first)
                assert text.find(end, i) > i, (f, end)
        bytes_, source = bench.captured_traffic(name)
        # either the capture still describes the kernel, or the line says why not
        assert (bytes_ is not None and source == c["profile"]) or \
            (bytes_ is None and "capture" in source)


if __name__ == "__main__":
    sys.exit(pytest.main([__file__, "-q"]))
