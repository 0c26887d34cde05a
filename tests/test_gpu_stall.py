"""Bounded waits that run out, on the GPU, without any fault.

Every mbarrier wait in the library's kernels gives up after a bound, raises an
abort flag, drains the copies it issued, frees its TMEM and records
JMOE_ETIMEOUT in the device error word.  jmoe_test_stall arms one forward call
in which a producer withholds its copies (the tensor-core GEMM's weight
producers stop before their first tile; the decode GEMV's first warp never
issues its first copy), with a short bound (about 1 ms), so the consumers'
waits run out.  The test checks the status, then that the next forward on the
same process is correct again.
"""
import numpy as np
import pytest

from layers import DeviceLayer, OracleLayer, assert_close, bf16_to_f64
from synth.workloads import TINY, Workload

torch = pytest.importorskip("torch")

import int8_weight_moe_b200 as jm  # noqa: E402

SHORT_WAIT = 2_000_000  # SM cycles, about 1 ms


WIDE = Workload("wide_stall", 18, 8, 8256, 128, E=4)


@pytest.mark.gpu
@pytest.mark.parametrize("target,path,wl", [(jm.JMOE_STALL_TENSOR_GEMM, jm.JMOE_PATH_PREFILL, TINY),
                                            (jm.JMOE_STALL_DECODE_GEMV, jm.JMOE_PATH_DECODE, TINY),
                                            (jm.JMOE_STALL_DECODE_GEMV, jm.JMOE_PATH_DECODE, WIDE)],
                         ids=["tensor_gemm", "decode_gemv", "decode_gemv_d8256"])
def test_wait_runs_out_then_next_call_is_correct(target, path, wl):
    dev, ora = DeviceLayer(wl), OracleLayer(wl)
    ids, g = jm.jmoe_route(dev.x, dev.w_router, wl.top_k, dev.bias)
    torch.cuda.synchronize()
    assert jm.jmoe_last_error() == jm.JMOE_OK
    jm.jmoe_test_stall(target, SHORT_WAIT)
    try:
        jm.jmoe_forward(dev.desc(path), dev.x, ids, g)
    finally:
        jm.jmoe_test_stall(0)
    assert jm.jmoe_last_error() == jm.JMOE_ETIMEOUT
    assert jm.jmoe_last_error() == jm.JMOE_OK  # cleared by the read

    out = jm.jmoe_forward(dev.desc(path), dev.x, ids, g)
    torch.cuda.synchronize()
    assert jm.jmoe_last_error() == jm.JMOE_OK
    _, io, go = ora.route()
    assert np.array_equal(ids.cpu().numpy(), io)
    assert_close(bf16_to_f64(out), ora.forward_tokens(np.arange(wl.T), io, go), "after stall")


@pytest.mark.gpu
def test_armed_stall_is_one_shot_and_disarmable():
    dev = DeviceLayer(TINY)
    ids, g = jm.jmoe_route(dev.x, dev.w_router, TINY.top_k, dev.bias)
    jm.jmoe_test_stall(jm.JMOE_STALL_DECODE_GEMV, SHORT_WAIT)
    jm.jmoe_test_stall(0)  # disarmed before any call
    ref = jm.jmoe_forward(dev.desc(jm.JMOE_PATH_DECODE), dev.x, ids, g)
    assert jm.jmoe_last_error() == jm.JMOE_OK
    jm.jmoe_test_stall(jm.JMOE_STALL_DECODE_GEMV, SHORT_WAIT)
    jm.jmoe_forward(dev.desc(jm.JMOE_PATH_DECODE), dev.x, ids, g)  # takes the stall
    assert jm.jmoe_last_error() == jm.JMOE_ETIMEOUT
    again = jm.jmoe_forward(dev.desc(jm.JMOE_PATH_DECODE), dev.x, ids, g)  # runs normally
    torch.cuda.synchronize()
    assert jm.jmoe_last_error() == jm.JMOE_OK
    assert torch.equal(again, ref)
