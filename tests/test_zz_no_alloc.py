"""The allocation-free forward, for callers that cannot allocate device memory
when they call the layer (a serving engine whose pool already owns all of
HBM, or a latency-critical path that cannot afford cudaMalloc's implicit
synchronisation).  Its scratch is a fixed array inside the library.

The checks go through the C ABI (ctypes): two calls in a row, on different
token batches, each compared bit for bit with the workspace-taking
jmoe_forward on the same inputs (both run the same deterministic decode
kernels, so any difference is a scratch-layout or stale-scratch fault), the
first batch also against the CPU oracle within the parity tolerance of the
other tests; and an oversized problem is refused before anything is
launched.  The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

import synth
from layers import DeviceLayer, OracleLayer, assert_close, bf16_to_f64
from synth.workloads import MINI_DECODE, Workload

torch = pytest.importorskip("torch")

import int8_weight_moe_b200 as jm  # noqa: E402

GOOD = 0x10000  # aligned fake address for argument-only checks (never dereferenced)


def _noalloc(desc, x, ids, w, out):
    return jm.load().jmoe_forward_noalloc(ctypes.byref(desc), x.data_ptr(), x.shape[0],
                                          ids.data_ptr(), w.data_ptr(), out.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_noalloc_matches_forward_on_two_calls_in_a_row():
    dev = DeviceLayer(MINI_DECODE)
    desc = dev.desc()
    batches = [dev.x, synth.normal_bf16_gpu(MINI_DECODE.seed + 100, synth.X, 1.0,
                                            tuple(dev.x.shape))]
    for i, x in enumerate(batches):
        ids, g = jm.jmoe_route(x, dev.w_router, MINI_DECODE.top_k)
        ref = jm.jmoe_forward(desc, x, ids, g)
        out = torch.full_like(x, float("nan"))
        assert _noalloc(desc, x, ids, g, out) == jm.JMOE_OK
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"batch {i}: noalloc differs from jmoe_forward"
        if i == 0:
            ora = OracleLayer(MINI_DECODE)
            _, io, go = ora.route()
            assert np.array_equal(ids.cpu().numpy(), io)
            assert_close(bf16_to_f64(out), ora.forward_tokens(np.arange(MINI_DECODE.T), io, go),
                         "noalloc vs oracle")
    assert jm.jmoe_last_error() == jm.JMOE_OK


@pytest.mark.gpu
def test_noalloc_refuses_problems_beyond_its_scratch():
    # Large-sized layer, 96 tokens top-2: the decode scratch would be ~56 MiB,
    # more than the fixed 32 MiB array; refused on the host, nothing launched.
    desc = jm.MoeDesc(16, 2, 8192, 24576, GOOD, GOOD, GOOD, GOOD, 0)
    too_big = jm.jmoe_forward_workspace_size(
        jm.MoeDesc(16, 2, 8192, 24576, GOOD, GOOD, GOOD, GOOD, jm.JMOE_PATH_DECODE), 96)
    assert too_big > jm.NOALLOC_SCRATCH_BYTES
    st = jm.load().jmoe_forward_noalloc(ctypes.byref(desc), GOOD, 96, GOOD, GOOD, GOOD, None)
    assert st == jm.JMOE_EWORKSPACE
    ok_size = jm.jmoe_forward_workspace_size(
        jm.MoeDesc(16, 2, 8192, 24576, GOOD, GOOD, GOOD, GOOD, jm.JMOE_PATH_DECODE), 32)
    assert ok_size <= jm.NOALLOC_SCRATCH_BYTES
