"""The C-ABI library on the host: it loads, exports every entry point the
header declares, and rejects bad arguments before launching anything.  No GPU
is needed: every call here fails validation (or is a pure size query), so no
CUDA call is reached."""
import ctypes
import re

import pytest

import int8_weight_moe_b200 as jm

BAD = 0x1001  # a misaligned fake address; never dereferenced (validation fails first)
GOOD = 0x10000  # an aligned fake address; only passed where another argument is invalid


def header_functions():
    with open(jm.HEADER) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"^(?:jmoe_status|const char\*)\s+(jmoe_\w+)\(", text, re.M)))


def test_library_exports_every_header_symbol():
    lib = jm.load()
    declared = header_functions()
    assert set(declared) == set(jm.EXPORTED)
    for name in declared:
        assert hasattr(lib, name), name


def test_cuda_error_string_is_per_thread_and_starts_empty():
    import threading

    got = []
    t = threading.Thread(target=lambda: got.append(jm.jmoe_cuda_error_string()))
    t.start()
    t.join()
    assert got == ["no CUDA error"]


def test_status_strings():
    for code in range(8):
        assert jm.status_string(code).startswith("JMOE_")
    assert "unknown" in jm.status_string(99)


def desc(**kw):
    d = dict(E=16, top_k=2, d_model=256, d_ff=512, w_gu=GOOD, s_gu=GOOD, w_d=GOOD, s_d=GOOD,
             path=0)
    d.update(kw)
    return jm.MoeDesc(**d)


def call_forward(dsc, x=GOOD, T=8, ids=GOOD, w=GOOD, out=GOOD, ws=GOOD, ws_bytes=1 << 30):
    return jm.load().jmoe_forward(ctypes.byref(dsc), x, T, ids, w, out, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(E=0), jm.JMOE_EUNSUPPORTED), (dict(E=65), jm.JMOE_EUNSUPPORTED),
    (dict(top_k=5), jm.JMOE_EUNSUPPORTED), (dict(E=1, top_k=2), jm.JMOE_EUNSUPPORTED),
    (dict(E=3, top_k=4), jm.JMOE_EUNSUPPORTED),
    (dict(d_model=100), jm.JMOE_EUNSUPPORTED), (dict(d_ff=96), jm.JMOE_EUNSUPPORTED),
    (dict(d_model=0), jm.JMOE_EINVAL), (dict(path=7), jm.JMOE_EINVAL),
    (dict(w_gu=None), jm.JMOE_EINVAL), (dict(s_d=None), jm.JMOE_EINVAL),
    (dict(w_d=BAD), jm.JMOE_EALIGN), (dict(s_gu=BAD), jm.JMOE_EALIGN),
])
def test_forward_rejects_bad_descriptor(kw, status):
    assert call_forward(desc(**kw)) == status


def test_forward_rejects_bad_buffers():
    assert call_forward(desc(), T=-1) == jm.JMOE_EINVAL
    assert call_forward(desc(), x=None) == jm.JMOE_EINVAL
    assert call_forward(desc(), out=BAD) == jm.JMOE_EALIGN
    assert call_forward(desc(), ids=BAD) == jm.JMOE_EALIGN
    assert call_forward(desc(), ws_bytes=16) == jm.JMOE_EWORKSPACE
    assert call_forward(desc(), ws=None) == jm.JMOE_EWORKSPACE
    assert call_forward(desc(), T=1 << 24) == jm.JMOE_EUNSUPPORTED
    # T = 0 is a no-op that succeeds without touching anything
    assert call_forward(desc(), T=0, x=None, ids=None, w=None, out=None, ws=None) == jm.JMOE_OK


def test_workspace_size_queries():
    small = jm.jmoe_forward_workspace_size(desc(path=jm.JMOE_PATH_DECODE), 8)
    big = jm.jmoe_forward_workspace_size(desc(path=jm.JMOE_PATH_DECODE), 64)
    assert 0 < small < big
    assert jm.jmoe_forward_workspace_size(desc(path=jm.JMOE_PATH_DECODE), 0) > 0
    with pytest.raises(jm.JmoeError):
        jm.jmoe_forward_workspace_size(desc(d_ff=100), 8)
    assert jm.jmoe_mlp_workspace_size(16, 256, 512, jm.JMOE_PATH_DECODE) > 0


def test_quantize_route_permute_validation():
    lib = jm.load()
    assert lib.jmoe_quantize(GOOD, 4, 12, GOOD, GOOD, None) == jm.JMOE_EUNSUPPORTED
    assert lib.jmoe_quantize(GOOD, -1, 16, GOOD, GOOD, None) == jm.JMOE_EINVAL
    assert lib.jmoe_quantize(None, 4, 16, GOOD, GOOD, None) == jm.JMOE_EINVAL
    assert lib.jmoe_quantize(BAD, 4, 16, GOOD, GOOD, None) == jm.JMOE_EALIGN
    assert lib.jmoe_quantize(None, 0, 16, None, None, None) == jm.JMOE_OK
    assert lib.jmoe_route(GOOD, 4, 256, GOOD, None, 65, 2, GOOD, GOOD, None, None) == \
        jm.JMOE_EUNSUPPORTED
    assert lib.jmoe_route(GOOD, 4, 256, GOOD, None, 64, 5, GOOD, GOOD, None, None) == \
        jm.JMOE_EUNSUPPORTED
    assert lib.jmoe_route_ex(GOOD, 4, 256, GOOD, None, 16, 2, 2, GOOD, GOOD, None, None) == \
        jm.JMOE_EINVAL
    assert lib.jmoe_route_ex(None, 0, 256, None, None, 64, 4, jm.JMOE_ROUTE_SOFTMAX_GATES, None,
                             None, None, None) == jm.JMOE_OK
    assert lib.jmoe_route(GOOD, 4, 100, GOOD, None, 16, 2, GOOD, GOOD, None, None) == \
        jm.JMOE_EUNSUPPORTED
    assert lib.jmoe_route(GOOD, 4, 256, GOOD, BAD, 16, 2, GOOD, GOOD, None, None) == \
        jm.JMOE_EALIGN
    assert lib.jmoe_route(None, 4, 256, GOOD, None, 16, 2, GOOD, GOOD, None, None) == \
        jm.JMOE_EINVAL
    assert lib.jmoe_route(None, 0, 256, None, None, 16, 2, None, None, None, None) == jm.JMOE_OK
    assert lib.jmoe_permute(GOOD, 4, 5, 16, GOOD, GOOD, GOOD, None) == jm.JMOE_EUNSUPPORTED
    assert lib.jmoe_permute(GOOD, 4, 2, 65, GOOD, GOOD, GOOD, None) == jm.JMOE_EUNSUPPORTED
    assert lib.jmoe_permute(GOOD, 4, 2, 16, None, GOOD, GOOD, None) == jm.JMOE_EINVAL
    assert lib.jmoe_permute(GOOD, 4, 2, 16, GOOD, BAD, GOOD, None) == jm.JMOE_EALIGN


def test_mlp_validation():
    lib = jm.load()
    args = [GOOD, 8, 256, 512, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 1 << 30, 0, None]
    bad_d = list(args); bad_d[2] = 200
    assert lib.jmoe_mlp_forward(*bad_d) == jm.JMOE_EUNSUPPORTED
    no_x = list(args); no_x[0] = None
    assert lib.jmoe_mlp_forward(*no_x) == jm.JMOE_EINVAL
    small = list(args); small[10] = 8
    assert lib.jmoe_mlp_forward(*small) == jm.JMOE_EWORKSPACE


def test_launch_counter_counts_nothing_for_rejected_calls():
    lib = jm.load()
    assert lib.jmoe_launch_count(None) == jm.JMOE_EINVAL
    n0 = jm.jmoe_launch_count()
    assert n0 >= 0
    assert lib.jmoe_quantize(None, 4, 16, GOOD, GOOD, None) == jm.JMOE_EINVAL
    assert lib.jmoe_permute(GOOD, 4, 2, 16, None, GOOD, GOOD, None) == jm.JMOE_EINVAL
    assert jm.jmoe_launch_count() == n0


def test_check_hook_is_unsupported_in_the_normal_build():
    # the normal build has no device checks: the hook refuses before any CUDA call
    assert jm.load().jmoe_test_check(None) == jm.JMOE_EUNSUPPORTED
    assert jm.status_string(jm.JMOE_EBOUNDS).startswith("JMOE_EBOUNDS")


def test_checks_build_exports_the_same_symbols():
    import ctypes
    import os

    if not os.path.exists(jm.CHECKS_LIB_PATH):
        pytest.skip("libjmoe_checks.so not built")
    lib = ctypes.CDLL(jm.CHECKS_LIB_PATH)
    for name in jm.EXPORTED:
        assert hasattr(lib, name), name


def test_stall_hook_validation():
    lib = jm.load()
    assert lib.jmoe_test_stall(3, 2_000_000) == jm.JMOE_EINVAL
    assert lib.jmoe_test_stall(-1, 2_000_000) == jm.JMOE_EINVAL
    assert lib.jmoe_test_stall(jm.JMOE_STALL_TENSOR_GEMM, 10) == jm.JMOE_EINVAL
    assert lib.jmoe_test_stall(jm.JMOE_STALL_DECODE_GEMV, 10 ** 10) == jm.JMOE_EINVAL
    assert lib.jmoe_test_stall(jm.JMOE_STALL_DECODE_GEMV, 2_000_000) == jm.JMOE_OK
    assert lib.jmoe_test_stall(0, 0) == jm.JMOE_OK  # disarms
