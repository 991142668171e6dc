"""Host checks of bench.py's accounting: the per-kernel algorithmic work of each forward path
plus the backward adds up to the step's 12pd flops (4pd forward, 8pd backward), for
non-causal and causal workloads and for the fp32 path; the executed work is never below the
algorithmic work; the phase and roofline arithmetic gives the fractions it should."""
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
    for kind, (alg, executed, nbytes) in model.items():
        assert executed >= alg and nbytes > 0, kind
    # the backward executes 14pd: S^T recomputed in the key-major kernel, S and dP in the
    # query-major one
    assert model["bwd_rows"][1] + model["bwd_keys"][1] == pytest.approx(total * 14 / 12)


def test_fp32_kernels_add_up_to_the_step():
    bench = _bench()
    w = bench.WORKLOADS["f32"]
    model = bench.kernel_model(w)
    kinds = ["f32_qk_slab", "slab_softmax", "f32_pv_ring_rows", "rowdot", "f32_bwd_slab",
             "f32_ring_keys", "f32_dq_ring_rows"]
    assert sum(model[k][0] for k in kinds) == pytest.approx(bench.step_flops(w))
    assert set(kinds) == bench.F32_KINDS


def test_causal_counts_the_live_triangle():
    bench = _bench()
    assert bench.live_entries(4, True) == 10 and bench.live_entries(4, False) == 16


def test_phase_fractions_and_end_to_end_roofline():
    """Two kernels with made-up durations: the per-kernel fractions are work / time / peak, the
    dominant kernel gives the roofline object, and the end-to-end fraction is the sum of the
    kernels' lower bounds over the step time."""
    bench = _bench()
    w = bench.WORKLOADS["long"]
    model = bench.kernel_model(w)
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1300.0,
             "source": "test"}
    cp = bench.compute_peaks(peaks, {"reasons": []}, 70.0)
    # 2 steps: bwd_keys 1 launch per step of 4 ms, qk_slab 10 launches per step of 0.3 ms each
    prof = {"bwd_keys": (8.0, 2), "qk_slab": (6.0, 20)}
    ph = bench.phases_from_profile(prof, 2, w, peaks, cp)
    assert [p["kernel"] for p in ph] == ["bwd_keys", "qk_slab"]
    bk, qk = ph
    assert bk["bound"] == "tensor" and qk["bound"] == "hbm"
    assert bk["achieved_tflops"] == pytest.approx(model["bwd_keys"][0] / 4e-3 / 1e12)
    assert bk["compute_frac"] == pytest.approx(bk["achieved_tflops"] / 1500.0)
    assert qk["alg_bytes_per_launch"] == pytest.approx(model["qk_slab"][2] / 10)
    assert qk["hbm_frac"] == pytest.approx(model["qk_slab"][2] / 3e-3 / 1e9 / 6000.0)
    roof = bench.roofline_of(ph, peaks, None)
    assert roof["kernel"] == "bwd_keys" and roof["unit"] == "TFLOP/s"
    assert roof["frac"] == pytest.approx(bk["compute_frac"])
    e2e = bench.roofline_e2e(ph, 10.0)
    lb = (model["bwd_keys"][0] / 1500e12 + model["qk_slab"][2] / 6000e9) * 1e3
    assert e2e["bound_ms"] == pytest.approx(lb)
    assert e2e["frac"] == pytest.approx(lb / 10.0)
    # under the power cap the sustained bf16 rate is the denominator
    capped = bench.compute_peaks(peaks, {"reasons": ["sw_power_cap"]}, 70.0)
    assert capped("bwd_keys")[0] == 1300.0 and capped("f32_qk_slab")[0] == 70.0


def test_row_sample_spreads_over_the_sequence():
    bench = _bench()
    rows = bench._sample_rows(16384, 5)
    assert rows[0] == 0 and rows[-1] == 16383 and len(rows) == 5
    w = dict(L=8, d=2, causal=True)
    assert bench._row_flops(w, [0, 7]) == 8.0 * (1 + 8) * 2


def test_slab_kernels_are_compared_with_their_direction():
    """The score kernel (writes) against the write probe, softmax/PV (reads) against the read
    probe; other kernels and a missing probe add nothing."""
    b = _bench()
    phases = [{"kernel": "qk_slab", "achieved_gbs": 5000.0},
              {"kernel": "pv_softmax", "achieved_gbs": 4800.0},
              {"kernel": "bwd_keys", "achieved_gbs": 500.0}]
    b.annotate_directions(phases, {"read": 6000.0, "write": 6250.0})
    assert phases[0]["hbm_frac_of_write_probe"] == pytest.approx(0.8)
    assert phases[1]["hbm_frac_of_read_probe"] == pytest.approx(0.8)
    assert not any(k.startswith("hbm_frac_of") for k in phases[2])
    fresh = [{"kernel": "qk_slab", "achieved_gbs": 5000.0}]
    b.annotate_directions(fresh, None)
    assert list(fresh[0]) == ["kernel", "achieved_gbs"]
