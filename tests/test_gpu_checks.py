"""The bounds-check build (libjmoe_checks.so: the same sources compiled with
JMOE_CHECKS=1) on the GPU.

Every device bounds check of that build raises a bit of the device error
word and skips its access instead of trapping; jmoe_last_error then returns
JMOE_EBOUNDS.  This is the library's stand-in for a memory checker: here the
checks build runs the layer over routings, shapes and paths that reach every
checked index (both grouping kernels, both expert paths, ragged tiles, 64
experts, the dense entry, the expert-parallel dispatch and combine) and must
report no failed check and give the same outputs as the normal build, bit for
bit.  The hook jmoe_test_check makes one check fail without touching memory,
which shows that a failure reaches jmoe_last_error.
"""
import contextlib

import pytest

from layers import DeviceLayer
from synth.workloads import TINY, Workload

torch = pytest.importorskip("torch")

import int8_weight_moe_b200 as jm  # noqa: E402

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def library(path):
    old_path, old_lib = jm.LIB_PATH, jm._lib
    jm.LIB_PATH, jm._lib = path, None
    try:
        yield
    finally:
        torch.cuda.synchronize()
        jm.LIB_PATH, jm._lib = old_path, old_lib


def both(fn):
    """fn() under the normal build, then under the checks build; returns both
    results and the checks build's error status."""
    with library(jm.LIB_PATH):
        ref = fn()
        torch.cuda.synchronize()
    with library(jm.CHECKS_LIB_PATH):
        assert jm.jmoe_last_error() in (jm.JMOE_OK, jm.JMOE_EBOUNDS)  # clear the word
        got = fn()
        torch.cuda.synchronize()
        status = jm.jmoe_last_error()
    return ref, got, status


def assert_same(ref, got):
    ref = ref if isinstance(ref, (tuple, list)) else (ref,)
    got = got if isinstance(got, (tuple, list)) else (got,)
    for r, g in zip(ref, got):
        assert torch.equal(r, g)


def test_check_hook_reaches_last_error():
    with library(jm.CHECKS_LIB_PATH):
        assert jm.jmoe_last_error() in (jm.JMOE_OK, jm.JMOE_EBOUNDS)
        assert jm.jmoe_test_check() == jm.JMOE_OK
        assert jm.jmoe_last_error() == jm.JMOE_EBOUNDS
        assert jm.jmoe_last_error() == jm.JMOE_OK  # read and cleared


CASES = [
    (TINY, jm.JMOE_PATH_DECODE), (TINY, jm.JMOE_PATH_PREFILL),
    (Workload("chk_ragged", 31, 37, 320, 576, bias=None), jm.JMOE_PATH_DECODE),
    (Workload("chk_ragged", 31, 37, 320, 576, bias=None), jm.JMOE_PATH_PREFILL),
    (Workload("chk_e64", 32, 37, 256, 576, E=64, top_k=4), jm.JMOE_PATH_DECODE),
    (Workload("chk_e64", 32, 300, 256, 576, E=64, top_k=4), jm.JMOE_PATH_PREFILL),
    (Workload("chk_wide", 33, 20, 1088, 192, E=4, bias=None), jm.JMOE_PATH_DECODE),
    (Workload("chk_big", 34, 1200, 256, 512), jm.JMOE_PATH_AUTO),
]


@pytest.mark.parametrize("wl,path", CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_layer_under_checks_is_clean_and_identical(wl, path):
    dev = DeviceLayer(wl)

    def run():
        ids, g = jm.jmoe_route(dev.x, dev.w_router, wl.top_k, dev.bias)
        out = jm.jmoe_forward(dev.desc(path), dev.x, ids, g)
        return ids, g, out

    ref, got, status = both(run)
    assert status == jm.JMOE_OK
    assert_same(ref, got)


def test_dense_permute_and_norm_under_checks():
    wl = Workload("chk_dense", 35, 300, 256, 512, E=1, top_k=1, dense=True)
    dev = DeviceLayer(wl)
    ref, got, status = both(lambda: jm.jmoe_mlp_forward(dev.x, dev.w_gu[0], dev.s_gu[0],
                                                         dev.w_d[0], dev.s_d[0]))
    assert status == jm.JMOE_OK
    assert_same(ref, got)
    ids = torch.randint(0, 16, (3000, 2), dtype=torch.int32, device="cuda")
    ref, got, status = both(lambda: jm.jmoe_permute(ids, 16))
    assert status == jm.JMOE_OK
    assert_same(ref, got)
    wl = Workload("chk_norm", 36, 40, 256, 512)
    dev = DeviceLayer(wl)
    gamma = torch.ones(256, dtype=torch.bfloat16, device="cuda")
    ref, got, status = both(lambda: jm.jmoe_rmsnorm_route(dev.x, gamma, 1e-6, dev.w_router, 2))
    assert status == jm.JMOE_OK
    assert_same(ref, got)


def test_expert_parallel_kernels_under_checks():
    wl = Workload("chk_ep", 37, 50, 256, 512, E=16, top_k=2)
    dev = DeviceLayer(wl)
    ids, gates = jm.jmoe_route(dev.x, dev.w_router, 2)

    def run():
        offsets, perm, inv, x_send, local_ids = jm.jmoe_ep_dispatch(dev.x, ids, 16, 4)
        out = jm.jmoe_ep_combine(x_send.contiguous(), inv, gates)
        return offsets, perm, inv, x_send, local_ids, out

    ref, got, status = both(run)
    assert status == jm.JMOE_OK
    assert_same(ref, got)
