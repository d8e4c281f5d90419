"""Host logic without a GPU: the sweep's per-layer checkpoint / resume, the shared-input block
layout, and the bench's roofline arithmetic and bounded oracle sample."""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

LAYERS = (("q", 8, 4, "attn"), ("k", 4, 4, "attn"), ("o", 8, 4, "o"), ("down", 4, 12, "down"))


def _inputs(block):
    g = torch.Generator().manual_seed(block)
    Ws = {name: torch.randn(m, n, generator=g) for name, m, n, _ in LAYERS}
    Xs = {"attn": torch.randn(5, 4, generator=g), "o": torch.randn(5, 4, generator=g),
          "down": torch.randn(5, 12, generator=g)}
    return Ws, Xs


def _fake_block(calls):
    """A stand-in for BlockQuantizer.run: deterministic outputs from the inputs."""
    def q(Ws, Xs, names):
        calls.append(tuple(names))
        out = {}
        for name, _, _, key in LAYERS:
            if name in names:
                out[name] = {"codes": (Ws[name] * 7).round().to(torch.int32),
                             "loss": (Ws[name] @ Xs[key].T).pow(2).sum().reshape(1)}
        return out
    return q


def test_sweep_resumes_at_the_first_missing_layer(tmp_path):
    from post_weight_quantization_22_b200.pipeline import SweepCheckpoint, run_sweep
    full = SweepCheckpoint(str(tmp_path / "full"), "cfg5")
    calls = []
    assert run_sweep(range(3), LAYERS, _inputs, _fake_block(calls), full) == 12
    assert len(calls) == 3

    part = SweepCheckpoint(str(tmp_path / "part"), "cfg5")
    seen = []

    class Stop(Exception):
        pass

    def stop_after_six(b, name):
        seen.append((b, name))
        if len(seen) == 6:
            raise Stop()
    calls2 = []
    with pytest.raises(Stop):
        run_sweep(range(3), LAYERS, _inputs, _fake_block(calls2), part, on_layer=stop_after_six)
    # a half-written file from a crash is not a result
    open(part.path(2, "q") + ".tmp", "wb").write(b"partial")
    calls3 = []
    assert run_sweep(range(3), LAYERS, _inputs, _fake_block(calls3), part) == 6
    assert calls3 == [("o", "down"), ("q", "k", "o", "down")]  # block 0 skipped entirely
    for b in range(3):
        for name, _, _, _ in LAYERS:
            a, c = full.load(b, name), part.load(b, name)
            assert torch.equal(a["codes"], c["codes"]) and torch.equal(a["loss"], c["loss"])
    # nothing left to do: no inputs are generated
    def no_inputs(b):
        raise AssertionError("regenerated a finished block")
    assert run_sweep(range(3), LAYERS, no_inputs, _fake_block([]), part) == 0


def test_sweep_block_inputs_share_one_input_per_kind():
    from post_weight_quantization_22_b200 import synth
    Ws, Xs = synth.sweep_block(0, scale=16)
    assert set(Xs) == {"attn", "o", "mlp", "down"}
    for name, m, n, kind in synth.SWEEP_LAYERS:
        assert tuple(Ws[name].shape) == (m // 16, n // 16)
        assert Xs[kind].shape[1] == n // 16 and Ws[name].dtype == torch.bfloat16
    # the attention input of block 0 is the one the q/k/v parity test builds by hand
    x_seed = synth.sweep_seeds(0, 0, "attn")[1]
    ref = synth.to_bf16(synth.make_x("calib", synth.SWEEP_T // 16, 4096 // 16, x_seed))
    assert torch.equal(ref, Xs["attn"])


def test_stage_model_fractions_are_floor_over_measured():
    sys.path.insert(0, ROOT)
    import bench
    peaks = dict(hbm_gbs=6000.0, bf16_tflops=1500.0, fp64_tflops=36.0, tf32_tflops=750.0,
                 fp32_tflops=70.0, int8_tops=3000.0)
    inputs, layers = [("x", 4096, 4096)], [("w", 4096, 4096, "x")]
    ms = {"hessian": 0.8, "factor": 3.0, "column_loop": 2.0}
    st, ov = bench.stage_model(inputs, layers, 4, 128, 2, peaks, ms)
    n, T, m = 4096, 4096, 4096
    h_floor = 2 * n * (n + 1) / 2 * T * bench.HESSIAN_DIGIT_PRODUCTS / 3000e12
    assert st["hessian"]["t_roof_ms"] == pytest.approx(h_floor * 1e3, rel=1e-3)
    macs, fp64 = bench.factor_work(n)
    f_floor = 2 * macs * bench.FACTOR_DIGIT_PRODUCTS / 3000e12 + fp64 / 36e12
    assert st["factor"]["t_roof_ms"] == pytest.approx(f_floor * 1e3, rel=1e-3)
    assert st["column_loop"]["t_roof_ms"] == pytest.approx(3 * m * n * n / 750e12 * 1e3, rel=1e-3)
    for k in ms:
        assert st[k]["frac"] == pytest.approx(st[k]["t_roof_ms"] / ms[k], rel=1e-3)
    assert ov["t_ms"] == pytest.approx(5.8)
    assert ov["frac_as_built"] == pytest.approx(
        sum(st[k]["t_roof_ms"] for k in ms) / 5.8, rel=1e-3)


def test_oracle_sample_scales_each_part_by_its_cost():
    sys.path.insert(0, ROOT)
    import bench
    rng = np.random.default_rng(0)
    X = rng.standard_normal((64, 48))
    W = 0.02 * rng.standard_normal((40, 48))
    t, det = bench.oracle_layer_sample([(X, [(W, 3, 0)])], tokens=32, n_sub=24, rows=8)
    assert t == pytest.approx(det["hessian_s"] + det["factor_s"] + det["loop_s"])
    assert 0 < det["measured_s"] < t       # every part is scaled up from a smaller sample


def test_factor_work_model_matches_the_library_split_policy():
    """bench.factor_work follows the factor's schedule: the split products start at the width
    where the factor's workspace gains its digit planes, and the two parts add up to 2 n^3 / 3."""
    sys.path.insert(0, ROOT)
    import bench
    from post_weight_quantization_22_b200 import gq as G
    n0 = bench.FACTOR_SPLIT_MIN_N
    jump = G.gq_prepare_workspace_size(n0) / n0 ** 2 - G.gq_prepare_workspace_size(n0 - 1) / (n0 - 1) ** 2
    assert jump > 2.0                        # ~3 n^2 bytes of digit planes appear at n0
    assert bench.factor_work(n0 - 1)[0] == 0.0
    for n in (n0, 4096, 14336):
        macs, fp64 = bench.factor_work(n)
        assert 2 * macs + fp64 == pytest.approx(2 * n ** 3 / 3, rel=1e-12)
    macs, fp64 = bench.factor_work(14336)
    assert 2 * macs / (2 * 14336 ** 3 / 3) > 0.9   # nearly all of the factor at that width


def test_stage_traffic_only_for_captured_single_layer_widths():
    sys.path.insert(0, ROOT)
    import bench
    one = [("w", 4096, 14336, "x")]
    got = bench.stage_traffic("factor", one, sweep=False)
    assert got is not None and got["bytes"] > 1e10          # the 14336-wide factor call
    assert bench.stage_traffic("factor", [("w", 4096, 4096, "x")], False)["bytes"] < got["bytes"]
    assert bench.stage_traffic("factor", [("w", 4096, 5000, "x")], False) is None
    assert bench.stage_traffic("column_loop", one, False) is None
    assert bench.stage_traffic("factor", one + one, False) is None
    assert bench.stage_traffic("factor", one, True) is None
