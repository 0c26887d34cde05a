"""bench.py's host arithmetic, on CPU: the bytes and FLOPs the roofline
divides by, the dequantisation work reported beside them (INT8 weight
conversions per step) for hand-made routings whose answers follow from the
tile rules by hand, and the per-step percentiles of the dominant kernel."""
import types

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import bench  # noqa: E402
from synth.workloads import MINI_DECODE, MINI_DENSE, TINY  # noqa: E402


def test_dequant_conversions_decode_passes():
    d, f = 64, 128
    unit = 3 * d * f
    # passes of up to 8 tokens: 1 -> 1, 8 -> 1, 9 -> 2, 17 -> 3; untouched experts add nothing
    assert bench.dequant_conversions([1, 8, 9, 0, 17], d, f, prefill=False) == 7 * unit
    assert bench.dequant_conversions([0, 0], d, f, prefill=False) == 0


def test_dequant_conversions_tensor_core_tiles():
    d, f = 64, 128
    unit = 3 * d * f
    # rows padded to 128, tiles of 512: 1 -> 128 -> 1, 128 -> 1, 129 -> 256 -> 1,
    # 513 -> 640 -> 2, 1100 -> 1152 -> 3
    assert bench.dequant_conversions([1, 128, 129, 513, 1100], d, f, prefill=True) == 8 * unit


def _fake_layer(wl, ids, prefill):
    lay = types.SimpleNamespace(wl=wl, ids=ids)
    lay.touched_experts = lambda: bench.Layer.touched_experts(lay)
    lay.expert_counts = lambda: bench.Layer.expert_counts(lay)
    lay.prefill_path = lambda: prefill
    return lay


def test_kernel_work_decode_routing():
    wl = MINI_DECODE  # T = 8, top-2, 16 experts
    d, f = wl.d_model, wl.d_ff
    ids = torch.tensor([[t, (t + 1) % 16] for t in range(wl.T)], dtype=torch.int32)
    w = bench.kernel_work(_fake_layer(wl, ids, prefill=False))
    assert w["touched"] == 9  # experts 0..8
    assert w["gate_up_bytes"] == 9 * 2 * f * d + wl.T * d * 2
    assert w["gate_up_flops"] == 4 * wl.A * d * f
    # every touched expert has at most 2 tokens: one pass each
    assert w["dequant"]["int8_conversions_per_step"] == 9 * 3 * d * f
    assert w["dequant"]["per_touched_weight"] == 1.0


def test_kernel_work_all_tokens_on_one_expert():
    wl = TINY  # T = 64, top-2
    ids = torch.zeros((wl.T, 2), dtype=torch.int32)
    ids[:, 1] = 1
    w = bench.kernel_work(_fake_layer(wl, ids, prefill=False))
    assert w["touched"] == 2
    # 64 tokens on each of two experts: 8 passes each
    assert w["dequant"]["per_touched_weight"] == 8.0


def test_kernel_work_dense_layer():
    wl = MINI_DENSE  # one expert, every token
    w = bench.kernel_work(_fake_layer(wl, None, prefill=True))
    assert w["touched"] == 1
    tiles = -(-(-(-wl.T // 128) * 128) // 512)
    assert w["dequant"]["int8_conversions_per_step"] == tiles * 3 * wl.d_model * wl.d_ff
    assert np.isclose(w["dequant"]["per_touched_weight"], tiles)


def test_step_percentiles():
    p = bench.step_percentiles([float(v) for v in range(1, 102)])  # 1..101
    assert p == {"median": 51.0, "p10": 11.0, "p90": 91.0}
    assert bench.step_percentiles([0.25]) == {"median": 0.25, "p10": 0.25, "p90": 0.25}
