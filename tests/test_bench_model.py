"""Host checks of bench.py's accounting: the per-kernel algorithmic work of each forward path
plus the backward adds up to the step's 12pd flops (4pd forward, 8pd backward), for
non-causal and causal workloads."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", ["bert", "gpt", "long"])
def test_kernel_flops_add_up_to_the_step(name):
    bench = _bench()
    w = bench.WORKLOADS[name]
    model = bench.kernel_model(w)
    total = bench.step_flops(w)
    backward = model["bwd_rows"][0] + model["bwd_keys"][0]
    slab = model["qk_slab"][0] + model["pv_softmax"][0]
    recompute = model["fwd_stats"][0] + model["fwd_pv"][0]
    assert slab + backward == pytest.approx(total)
    assert recompute + backward == pytest.approx(total)
    assert backward == pytest.approx(2 * slab)  # 8pd against 4pd


def test_causal_counts_the_live_triangle():
    bench = _bench()
    assert bench.live_entries(4, True) == 10 and bench.live_entries(4, False) == 16
