"""CUDA path vs the CPU oracle, on the same seeded inputs, through the C ABI.

Bit-exact: INT8 weights and scales, router logits and top-k ids, the
permutation.  Floating-point outputs: max |d| <= 2e-2 max |ref| and
sum |d| / sum |ref| <= 5e-3 (bf16 I/O, fp32 accumulation); gates within 1e-6.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from exact import bf16_bits
from layers import (DeviceLayer, OracleLayer, assert_close, bf16_to_f64, boundary_tokens,
                    gate_sum_bound)
from synth.workloads import (LARGE_DECODE, LARGE_PREFILL_SKEW, MINI_DECODE, MINI_DECODE_E64,
                             MINI_DENSE, MINI_PREFILL, TINY, Workload)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import int8_weight_moe_b200 as jm  # noqa: E402

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def cuda_bf16(bits: np.ndarray):
    return torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).cuda()


# ----------------------------------------------------------------------------- quantisation


def test_quantize_golden_rows_bitexact():
    with open(os.path.join(GOLDEN, "quantize_rows.json")) as fh:
        rows = json.load(fh)["rows"]
    for row in rows:
        vals = np.array(row["values"], dtype=np.float32)
        pad = (-len(vals)) % 8  # the device kernel wants 16-byte rows
        bits = bf16_bits(np.concatenate([vals, np.zeros(pad, np.float32)]))[None, :]
        q, s = jm.jmoe_quantize(cuda_bf16(bits))
        qo, so = oracle.quantize(bits)
        assert np.array_equal(q.cpu().numpy(), qo), row["name"]
        assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32)), row["name"]


def test_quantize_tiny_all_weights_bitexact():
    dev = DeviceLayer(TINY)
    ora = OracleLayer(TINY)
    for e in range(TINY.E):
        qg, sg, qd, sd = ora.expert(e)
        assert np.array_equal(dev.w_gu[e].cpu().numpy(), qg)
        assert np.array_equal(dev.s_gu[e].cpu().numpy().view(np.uint32), sg.view(np.uint32))
        assert np.array_equal(dev.w_d[e].cpu().numpy(), qd)
        assert np.array_equal(dev.s_d[e].cpu().numpy().view(np.uint32), sd.view(np.uint32))


@pytest.mark.parametrize("wl", [MINI_DECODE, LARGE_DECODE], ids=lambda w: w.name)
def test_quantize_full_size_sampled_rows_bitexact(wl):
    """Full-size expert matrices quantised on the GPU; 3 experts x 48 sampled
    rows of each matrix re-derived by the oracle."""
    dev = DeviceLayer(wl, T=8)
    ora = OracleLayer(wl, T=8)
    rng = np.random.default_rng(0)
    f, d = wl.d_ff, wl.d_model
    for e in (0, wl.E // 2, wl.E - 1):
        for r in rng.integers(0, 2 * f, size=48):
            q, s = oracle.quantize(ora.gate_up_rows(e, int(r), 1))
            assert np.array_equal(dev.w_gu[e, r].cpu().numpy(), q[0])
            assert dev.s_gu[e, r].item() == s[0]
        for r in rng.integers(0, d, size=48):
            q, s = oracle.quantize(ora.down_rows(e, int(r), 1))
            assert np.array_equal(dev.w_d[e, r].cpu().numpy(), q[0])
            assert dev.s_d[e, r].item() == s[0]


def test_quantize_roundtrip_bound_on_device():
    w = synth.normal_bf16_gpu(77, synth.WD, 0.02, (512, 1024))
    q, s = jm.jmoe_quantize(w)
    wv = w.float().double()
    err = (wv - q.double() * s.double()[:, None]).abs()
    assert bool((err <= s.double()[:, None] / 2 * (1 + 2.0 ** -16)).all())
    assert int(q.abs().max(dim=1).values.min()) == 127


# ----------------------------------------------------------------------------- router


@pytest.mark.parametrize("wl", [TINY, MINI_DECODE, LARGE_DECODE, MINI_PREFILL, LARGE_PREFILL_SKEW],
                         ids=lambda w: w.name)
def test_route_bitexact(wl):
    dev = DeviceLayer(Workload(wl.name, wl.index, wl.T, wl.d_model, 64, wl.E, wl.top_k, wl.bias))
    ora = OracleLayer(wl)
    ids, g, logits = jm.jmoe_route(dev.x, dev.w_router, wl.top_k, dev.bias, want_logits=True)
    lo, io, go = ora.route()
    assert np.array_equal(logits.cpu().numpy().view(np.uint32), lo.view(np.uint32))
    assert np.array_equal(ids.cpu().numpy(), io)
    gg = g.cpu().numpy().astype(np.float64)
    assert np.abs(gg - go).max() <= 1e-6
    assert np.abs(gg.sum(axis=1) - 1.0).max() <= gate_sum_bound(wl.top_k)
    if wl.bias is not None:
        frac = float(np.isin(io, [0, 1]).mean())
        assert 0.33 <= frac <= 0.47, frac


@pytest.mark.parametrize("T,d,E", [(3, 12288, 16), (5, 16384, 12)])
def test_route_wide_rows_bitexact(T, d, E):
    # rows too wide for the per-token cluster kernel take the chunked one
    wl = Workload("route_wide", 13, T, d, 64, E=E)
    dev = DeviceLayer(wl)
    ora = OracleLayer(wl)
    ids, g, logits = jm.jmoe_route(dev.x, dev.w_router, wl.top_k, dev.bias, want_logits=True)
    lo, io, go = ora.route()
    assert np.array_equal(logits.cpu().numpy().view(np.uint32), lo.view(np.uint32))
    assert np.array_equal(ids.cpu().numpy(), io)
    assert np.abs(g.cpu().numpy().astype(np.float64) - go).max() <= 1e-6


@pytest.mark.parametrize("norm", [False, True], ids=["route", "rmsnorm_route"])
def test_route_mid_tokens_wide_rows_bitexact(norm):
    # 800 tokens of width 8192: fewer than the tiled kernel's usual threshold,
    # but the tiles are cheaper than one cluster per token at this width
    T, d, E = 800, 8192, 16
    x = synth.normal_bf16_gpu(25, synth.X, 1.0, (T, d))
    wr = synth.normal_f32_gpu(26, synth.WR, 0.02, (E, d))
    xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
    if norm:
        gam = (synth.normal_bf16_gpu(27, synth.X, 0.25, (d,)).float() + 1.0).to(torch.bfloat16)
        xn, ids, g, logits = jm.jmoe_rmsnorm_route(x, gam, 1e-6, wr, 2, want_logits=True)
        torch.cuda.synchronize()
        xb = oracle.rmsnorm(xb, gam.view(torch.int16).cpu().numpy().view(np.uint16), 1e-6)
        assert np.array_equal(xn.view(torch.int16).cpu().numpy().view(np.uint16), xb)
    else:
        ids, g, logits = jm.jmoe_route(x, wr, 2, None, want_logits=True)
        torch.cuda.synchronize()
    lo, io, go = oracle.route(xb, wr.cpu().numpy(), 2, None)
    assert np.array_equal(logits.cpu().numpy().view(np.uint32), lo.view(np.uint32))
    assert np.array_equal(ids.cpu().numpy(), io)
    assert np.abs(g.cpu().numpy().astype(np.float64) - go).max() <= 1e-6


def test_route_top1_and_ties():
    d, E = 256, 16
    x = synth.normal_bf16_gpu(3, synth.X, 1.0, (40, d))
    wr = synth.normal_f32_gpu(3, synth.WR, 0.02, (E, d))
    wr[7] = wr[3]
    bias = torch.zeros(E, dtype=torch.float32, device="cuda")
    bias[3] = bias[7] = 4.0
    ids, g = jm.jmoe_route(x, wr, 2, bias)
    assert bool((ids[:, 0] == 3).all()) and bool((ids[:, 1] == 7).all())
    assert bool((g == 0.5).all())
    ids1, g1 = jm.jmoe_route(x, wr, 1, None)
    _, io, _ = oracle.route(x.view(torch.int16).cpu().numpy().view(np.uint16),
                            wr.cpu().numpy(), 1, None)
    assert np.array_equal(ids1.cpu().numpy(), io)
    assert bool((g1 == 1.0).all())
    z = torch.zeros((4, d), dtype=torch.bfloat16, device="cuda")
    idz, gz = jm.jmoe_route(z, wr, 2, None)
    assert idz.cpu().numpy().tolist() == [[0, 1]] * 4 and bool((gz == 0.5).all())


def test_route_many_tokens_special_values():
    # Many tokens (the tiled kernel) with the values its exact rescaling of the
    # products has to get right: zero, subnormal, infinite and NaN token values
    # (one infinity only in the second 256-wide chunk), zero and subnormal router
    # weights, weights at the top of the fp32 range, and a ragged last chunk.
    T, d, E = 1300, 576, 16
    x = synth.normal_bf16_gpu(21, synth.X, 1.0, (T, d))
    wr = synth.normal_f32_gpu(22, synth.WR, 0.02, (E, d))
    xi = x.view(torch.int16)
    x[5] = 0.0
    xi[6, 1::2] = -32768                                  # -0.0
    sub = torch.arange(1, 128, dtype=torch.int16, device="cuda")
    xi[7, :127] = sub                                     # bf16 subnormals
    xi[7, 127:254] = sub | -32768
    xi[7, 254:] = 0
    x[9, 100] = float("inf")
    x[11, 3] = float("nan")
    x[13, 10], x[13, 200] = float("-inf"), float("inf")
    x[15, 300] = float("inf")                             # second chunk only
    x[1299, 570] = float("-inf")                          # last token, ragged chunk
    wr[2] = 0.0
    wr[4, ::3] = 1.0e-40                                  # fp32 subnormals
    wr[4, 1::3] = -3.0e-45
    x[:, [5, 7, 17]] *= 0.25                             # keeps the logits below the fp32 limit
    wr[6, 5], wr[8, 7], wr[9, 17] = 3.0e38, -3.3e38, 2.0 ** 127
    ids, g, logits = jm.jmoe_route(x, wr, 2, None, want_logits=True)
    torch.cuda.synchronize()
    lo, io, go = oracle.route(x.view(torch.int16).cpu().numpy().view(np.uint16),
                              wr.cpu().numpy(), 2, None)
    lg = logits.cpu().numpy()
    nan = np.isnan(lo)
    assert nan[11].all() and not nan[5].any() and not nan[7].any()
    # NaN payloads are not part of the method; where the logit is a number it
    # must match bit for bit
    assert np.array_equal(np.isnan(lg), nan)
    assert np.array_equal(lg[~nan].view(np.uint32), lo[~nan].view(np.uint32))
    assert np.array_equal(ids.cpu().numpy(), io)
    fin = np.isfinite(go).all(axis=1)
    assert fin.sum() >= T - 5
    assert np.abs(g.cpu().numpy().astype(np.float64)[fin] - go[fin]).max() <= 1e-6


@pytest.mark.parametrize("T,d", [(8, 576), (4, 12288)], ids=["cluster", "wide_rows"])
def test_route_few_tokens_special_values(T, d):
    # The same special values through the few-token routers (one token row
    # each: zeros and subnormals, +inf, NaN, -inf with +inf, ...), against the
    # oracle: logits bit for bit where they are numbers, NaN where it is NaN.
    E = 16
    x = synth.normal_bf16_gpu(23, synth.X, 1.0, (T, d))
    wr = synth.normal_f32_gpu(24, synth.WR, 0.02, (E, d))
    xi = x.view(torch.int16)
    sub = torch.arange(1, 128, dtype=torch.int16, device="cuda")
    xi[0, :127] = sub
    xi[0, 127:254] = sub | -32768
    xi[0, 254:] = 0
    x[1, d - 3] = float("inf")
    x[2, 5] = float("nan")
    x[3, 7], x[3, d // 2] = float("-inf"), float("inf")
    if T > 4:
        x[4] = 0.0
        xi[5, 1::2] = -32768
    wr[2] = 0.0
    wr[4, ::3] = 1.0e-40
    wr[4, 1::3] = -3.0e-45
    x[:, [9, 11]] *= 0.25
    wr[6, 9], wr[9, 11] = 3.0e38, 2.0 ** 127
    ids, g, logits = jm.jmoe_route(x, wr, 2, None, want_logits=True)
    torch.cuda.synchronize()
    lo, io, go = oracle.route(x.view(torch.int16).cpu().numpy().view(np.uint16),
                              wr.cpu().numpy(), 2, None)
    lg = logits.cpu().numpy()
    nan = np.isnan(lo)
    assert nan[2].all() and not nan[0].any()
    assert np.array_equal(np.isnan(lg), nan)
    assert np.array_equal(lg[~nan].view(np.uint32), lo[~nan].view(np.uint32))
    assert np.array_equal(ids.cpu().numpy(), io)
    fin = np.isfinite(go).all(axis=1)
    assert fin[0] and np.abs(g.cpu().numpy().astype(np.float64)[fin] - go[fin]).max() <= 1e-6


# ----------------------------------------------------------------------------- permutation


@pytest.mark.parametrize("T,k,E,mode", [(64, 2, 16, "uniform"), (37, 2, 16, "skew"),
                                         (1, 2, 16, "uniform"), (5000, 2, 16, "skew"),
                                         (16384, 2, 16, "uniform"), (300, 1, 1, "uniform"),
                                         (129, 2, 16, "one"), (200, 4, 64, "uniform"),
                                         (512, 2, 16, "skew"), (1025, 1, 40, "uniform"),
                                         (33, 1, 40, "skew"), (7, 3, 64, "one")])
def test_permute_bitexact(T, k, E, mode):
    """Up to 1024 assignments one warp sorts, above that the whole block: both
    sides of that boundary, 33 to 64 experts (two per lane) and ragged chunks."""
    rng = np.random.default_rng(T + k + E)
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    if mode == "skew":
        ids[:, 0] = np.minimum(ids[:, 0], 1)
    if mode == "one":
        ids[:] = 5
    off, perm, inv = jm.jmoe_permute(torch.from_numpy(ids).cuda(), E)
    oo, po, io = oracle.permute(ids, E)
    assert np.array_equal(off.cpu().numpy(), oo)
    assert np.array_equal(perm.cpu().numpy(), po)
    assert np.array_equal(inv.cpu().numpy(), io)


@pytest.mark.parametrize("T,k,E", [(40, 2, 16), (900, 2, 40), (3000, 2, 16)])
def test_permute_leaves_out_invalid_ids(T, k, E):
    """Ids outside [0, E) take no slot (inv = -1) and raise the device error
    word; the valid ones are grouped exactly as a stable sort of them alone
    (numpy's stable argsort here), on the warp path and the block path."""
    assert jm.jmoe_last_error() in (jm.JMOE_OK, jm.JMOE_EDEVICE)
    rng = np.random.default_rng(T * 7 + E)
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    flat = ids.reshape(-1)
    bad = rng.choice(flat.size, size=max(3, flat.size // 50), replace=False)
    flat[bad] = rng.choice(np.array([-1, E, 99, -7], dtype=np.int32), size=bad.size)
    off, perm, inv = jm.jmoe_permute(torch.from_numpy(ids).cuda(), E)
    torch.cuda.synchronize()
    assert jm.jmoe_last_error() == jm.JMOE_EDEVICE
    valid = (flat >= 0) & (flat < E)
    want_perm = np.flatnonzero(valid)[np.argsort(flat[valid], kind="stable")]
    want_off = np.concatenate([[0], np.cumsum(np.bincount(flat[valid], minlength=E))])
    want_inv = np.full(flat.size, -1, dtype=np.int64)
    want_inv[want_perm] = np.arange(want_perm.size)
    n = want_perm.size
    assert np.array_equal(off.cpu().numpy(), want_off)
    assert np.array_equal(perm.cpu().numpy()[:n], want_perm)
    assert np.array_equal(inv.cpu().numpy(), want_inv)


# ----------------------------------------------------------------------------- forward


def run_layer(dev, path=0):
    ids, g = jm.jmoe_route(dev.x, dev.w_router, dev.wl.top_k, dev.bias)
    out = jm.jmoe_forward(dev.desc(path), dev.x, ids, g)
    torch.cuda.synchronize()
    return ids, g, out


PATHS = [jm.JMOE_PATH_DECODE, jm.JMOE_PATH_PREFILL, jm.JMOE_PATH_AUTO]


@pytest.mark.parametrize("path", PATHS)
def test_forward_tiny_all_tokens(path):
    dev, ora = DeviceLayer(TINY), OracleLayer(TINY)
    ids, g, out = run_layer(dev, path)
    _, io, go = ora.route()
    assert np.array_equal(ids.cpu().numpy(), io)
    ref = ora.forward_tokens(np.arange(TINY.T), io, go)
    assert_close(bf16_to_f64(out), ref, "tiny")
    if path == jm.JMOE_PATH_PREFILL:
        assert jm.jmoe_last_error() == jm.JMOE_OK  # no bounded wait ran out


def test_forward_mini_decode_all_tokens():
    dev, ora = DeviceLayer(MINI_DECODE), OracleLayer(MINI_DECODE)
    ids, g, out = run_layer(dev)
    _, io, go = ora.route()
    assert np.array_equal(ids.cpu().numpy(), io)
    ref = ora.forward_tokens(np.arange(MINI_DECODE.T), io, go)
    assert_close(bf16_to_f64(out), ref, "mini decode")


def test_forward_large_decode_all_tokens():
    # every token of the batch: all touched experts (about 15 of 16) and every
    # 8-token pass of the decode kernels are compared
    dev, ora = DeviceLayer(LARGE_DECODE), OracleLayer(LARGE_DECODE)
    ids, g, out = run_layer(dev)
    _, io, go = ora.route()
    assert np.array_equal(ids.cpu().numpy(), io)
    assert np.unique(io).size >= 10
    tokens = np.arange(LARGE_DECODE.T)
    ref = ora.forward_tokens(tokens, io, go)
    assert_close(bf16_to_f64(out), ref, "large decode")


def test_forward_e64_top4_all_tokens():
    # Mini sizes with 64 experts and top-4, the bench's launch configuration
    dev, ora = DeviceLayer(MINI_DECODE_E64), OracleLayer(MINI_DECODE_E64)
    ids, g, out = run_layer(dev)
    _, io, go = ora.route()
    assert np.array_equal(ids.cpu().numpy(), io)
    assert np.allclose(g.cpu().numpy(), go, rtol=0, atol=4e-6)
    tokens = np.arange(MINI_DECODE_E64.T)
    ref = ora.forward_tokens(tokens, io, go)
    assert_close(bf16_to_f64(out), ref, MINI_DECODE_E64.name)


@pytest.mark.parametrize("wl", [MINI_PREFILL, LARGE_PREFILL_SKEW],
                         ids=["mini_prefill", "large_prefill_skewed"])
def test_forward_prefill_tile_boundaries(wl):
    """Full-size prefill, compared on the tokens whose assignments sit at each
    expert's first and last grouped row and on both sides of every 128-row
    boundary of every expert (the hot experts 0 and 1 of the skewed workload
    included), plus the first and last token of the batch."""
    dev, ora = DeviceLayer(wl), OracleLayer(wl)
    ids, g, out = run_layer(dev)
    _, io, go = ora.route()
    assert np.array_equal(ids.cpu().numpy(), io)
    tokens = sorted(set(boundary_tokens(io, wl.E, wl.top_k)) | {0, wl.T - 1})
    assert len(tokens) >= 4 * wl.E
    ref = ora.forward_tokens(tokens, io, go)
    got = bf16_to_f64(out)[tokens]
    assert_close(got, ref, wl.name)
    # every sampled row on its own, so no single bad row hides in the totals
    for i, t in enumerate(tokens):
        assert_close(got[i:i + 1], ref[i:i + 1], f"{wl.name} token {t}")


@pytest.mark.parametrize("path", PATHS)
def test_dense_mlp_tiny(path):
    wl = Workload("tiny_dense", 0, 64, 256, 512, E=1, top_k=1, dense=True)
    dev, ora = DeviceLayer(wl), OracleLayer(wl)
    out = jm.jmoe_mlp_forward(dev.x, dev.w_gu[0], dev.s_gu[0], dev.w_d[0], dev.s_d[0], path=path)
    torch.cuda.synchronize()
    assert_close(bf16_to_f64(out), ora.dense_forward_tokens(np.arange(64)), "tiny dense")


def test_dense_mlp_mini_tile_boundaries():
    # both rows on either side of every 128-row boundary, and the last row
    dev, ora = DeviceLayer(MINI_DENSE), OracleLayer(MINI_DENSE)
    out = jm.jmoe_mlp_forward(dev.x, dev.w_gu[0], dev.s_gu[0], dev.w_d[0], dev.s_d[0])
    torch.cuda.synchronize()
    T = MINI_DENSE.T
    tokens = sorted({0, T - 1} | {b + o for b in range(128, T, 128) for o in (-1, 0)})
    got, ref = bf16_to_f64(out)[tokens], ora.dense_forward_tokens(tokens)
    assert_close(got, ref, "mini dense")
    for i, t in enumerate(tokens):
        assert_close(got[i:i + 1], ref[i:i + 1], f"mini dense token {t}")


# ----------------------------------------------------------------------------- edge cases


@pytest.mark.parametrize("T,d,f", [(1, 256, 576), (2, 256, 576), (37, 320, 576),
                                   (129, 256, 576), (300, 320, 448)])
@pytest.mark.parametrize("path", PATHS)
def test_forward_ragged_token_counts(T, d, f, path):
    """Ragged token counts and ragged N tiles (d_model 320 is not a multiple of
    the 256-wide down tile, d_ff 576 / 448 not of the 128-channel gate/up tile)."""
    wl = Workload(f"ragged_T{T}_d{d}_f{f}", 7, T, d, f, bias=None)
    dev, ora = DeviceLayer(wl), OracleLayer(wl)
    ids, g, out = run_layer(dev, path)
    _, io, go = ora.route()
    assert np.array_equal(ids.cpu().numpy(), io)
    assert_close(bf16_to_f64(out), ora.forward_tokens(np.arange(T), io, go), f"T={T}")


@pytest.mark.parametrize("T,d,f", [(8, 1088, 192), (20, 4096, 128), (8, 8192, 128),
                                   (8, 8256, 128)], ids=lambda v: str(v))
def test_decode_gate_up_widths(T, d, f):
    """The decode path over d_model: 17, 64, 128 and 129 k-blocks of 64 (the
    K pieces of the split-K GEMV and the 4-D gate/up box walk them), with
    20 tokens in 8-token passes, the last one ragged."""
    wl = Workload(f"gu_T{T}_d{d}_f{f}", 16, T, d, f, E=4, bias=None)
    dev, ora = DeviceLayer(wl), OracleLayer(wl)
    ids, g, out = run_layer(dev, jm.JMOE_PATH_DECODE)
    assert jm.jmoe_last_error() == jm.JMOE_OK
    _, io, go = ora.route()
    assert np.array_equal(ids.cpu().numpy(), io)
    assert_close(bf16_to_f64(out), ora.forward_tokens(np.arange(T), io, go), wl.name)


@pytest.mark.parametrize("path", PATHS)
def test_forced_routing_one_expert_and_zero_input(path):
    wl = Workload("forced", 8, 200, 256, 512)
    dev, ora = DeviceLayer(wl), OracleLayer(wl)
    ids = np.full((wl.T, 2), 5, dtype=np.int32)
    ids[::3, 1] = 9
    gates = np.tile(np.array([0.75, 0.25], dtype=np.float32), (wl.T, 1))
    out = jm.jmoe_forward(dev.desc(path), dev.x, torch.from_numpy(ids).cuda(),
                          torch.from_numpy(gates).cuda())
    torch.cuda.synchronize()
    ref = ora.forward_tokens(np.arange(wl.T), ids, gates.astype(np.float64))
    assert_close(bf16_to_f64(out), ref, "forced")
    zero = torch.zeros_like(dev.x)
    outz = jm.jmoe_forward(dev.desc(path), zero, torch.from_numpy(ids).cuda(),
                           torch.from_numpy(gates).cuda())
    torch.cuda.synchronize()
    assert bool((outz.float() == 0).all())


def test_forward_top1_and_single_expert():
    wl = Workload("top1", 9, 50, 256, 512, E=16, top_k=1)
    dev, ora = DeviceLayer(wl), OracleLayer(wl)
    ids, g, out = run_layer(dev)
    _, io, go = ora.route()
    assert np.array_equal(ids.cpu().numpy(), io)
    assert_close(bf16_to_f64(out), ora.forward_tokens(np.arange(wl.T), io, go), "top1")
    wl1 = Workload("E1", 10, 30, 256, 512, E=1, top_k=1)
    dev1, ora1 = DeviceLayer(wl1), OracleLayer(wl1)
    ids1, g1, out1 = run_layer(dev1)
    assert bool((ids1 == 0).all()) and bool((g1 == 1).all())
    assert_close(bf16_to_f64(out1), ora1.dense_forward_tokens(np.arange(30)), "E=1")


def test_zero_tokens_is_a_noop():
    dev = DeviceLayer(TINY, T=1)
    x = dev.x[:0]
    ids = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    g = torch.empty((0, 2), dtype=torch.float32, device="cuda")
    out = jm.jmoe_forward(dev.desc(), x, ids, g)
    assert out.shape == (0, TINY.d_model)


# ----------------------------------------------------------------------------- invariants


@pytest.mark.parametrize("path", PATHS)
def test_token_permutation_and_determinism(path):
    wl = Workload("perm", 11, 96, 256, 512)
    dev = DeviceLayer(wl)
    ids, g, out = run_layer(dev, path)
    _, _, out2 = run_layer(dev, path)
    assert torch.equal(out, out2)  # run-to-run bitwise identical
    tp = torch.randperm(wl.T, generator=torch.Generator().manual_seed(0)).cuda()
    outp = jm.jmoe_forward(dev.desc(path), dev.x[tp].contiguous(), ids[tp].contiguous(),
                           g[tp].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(outp, out[tp])


@pytest.mark.parametrize("path", [jm.JMOE_PATH_DECODE, jm.JMOE_PATH_PREFILL])
def test_invalid_expert_id_sets_device_error_word(path):
    # A slot whose expert id is out of range takes no part in the layer: the
    # device error word is raised, and the token keeps its other slots (the
    # same result as a valid slot with gate 0, up to the order of the rows)
    assert jm.jmoe_last_error() in (jm.JMOE_OK, jm.JMOE_EDEVICE)
    dev = DeviceLayer(Workload("bad", 12, 8, 256, 512))
    ids = torch.full((8, 2), 1, dtype=torch.int32, device="cuda")
    ids[:, 0] = torch.arange(8, dtype=torch.int32, device="cuda") % 4 + 2
    ids[3, 1] = 99
    g = torch.full((8, 2), 0.5, dtype=torch.float32, device="cuda")
    out = jm.jmoe_forward(dev.desc(path), dev.x, ids, g)
    assert jm.jmoe_last_error() == jm.JMOE_EDEVICE
    assert jm.jmoe_last_error() == jm.JMOE_OK  # cleared by the read
    assert bool(torch.isfinite(out.float()).all())
    ids_ok, g_ok = ids.clone(), g.clone()
    ids_ok[3, 1], g_ok[3, 1] = 1, 0.0
    ref = jm.jmoe_forward(dev.desc(path), dev.x, ids_ok, g_ok)
    torch.cuda.synchronize()
    assert jm.jmoe_last_error() == jm.JMOE_OK
    assert_close(bf16_to_f64(out), bf16_to_f64(ref), "invalid slot left out")


def test_automatic_path_follows_the_measured_crossings():
    # decode kernels below 26 assignments per expert at d_model 4096, 21 at
    # 8192, linear in between (24 at 6144); 16 experts, top-2.  Only size
    # queries: nothing is launched.
    fake = 0x10000
    for d, f, t_switch in ((4096, 14336, 208), (6144, 16384, 192), (8192, 24576, 168)):
        desc = jm.MoeDesc(16, 2, d, f, fake, fake, fake, fake, jm.JMOE_PATH_AUTO)
        assert not jm.uses_prefill_path(desc, t_switch - 1), (d, t_switch - 1)
        assert jm.uses_prefill_path(desc, t_switch), (d, t_switch)
    dense = jm.MoeDesc(1, 1, 4096, 14336, fake, fake, fake, fake, jm.JMOE_PATH_AUTO)
    assert not jm.uses_prefill_path(dense, 127) and jm.uses_prefill_path(dense, 128)


@pytest.mark.parametrize("path,expected", [(jm.JMOE_PATH_DECODE, 6), (jm.JMOE_PATH_PREFILL, 5)])
def test_launch_counter_per_path(path, expected):
    # decode: grouping with fp16 token rows, gate/up GEMV, SwiGLU, fp16 hidden
    # rows, down GEMV, combine; tensor-core: grouping, row gather, two grouped
    # GEMMs, finalize.  The router is one more launch.
    dev = DeviceLayer(TINY)
    ids, g = jm.jmoe_route(dev.x, dev.w_router, TINY.top_k, dev.bias)
    n0 = jm.jmoe_launch_count()
    jm.jmoe_route(dev.x, dev.w_router, TINY.top_k, dev.bias, topk_ids=ids, topk_w=g)
    n1 = jm.jmoe_launch_count()
    jm.jmoe_forward(dev.desc(path), dev.x, ids, g)
    n2 = jm.jmoe_launch_count()
    torch.cuda.synchronize()
    assert (n1 - n0, n2 - n1) == (1, expected)


# ----------------------------------------------------------------------------- generalised routing

ROUTE_SHAPES = [(64, 4), (8, 2), (32, 3), (64, 1)]


@pytest.mark.parametrize("E,top_k", ROUTE_SHAPES, ids=lambda v: str(v))
@pytest.mark.parametrize("softmax_gates", [False, True], ids=["renorm", "softmax"])
@pytest.mark.parametrize("T,d", [(37, 256), (5, 12288), (1300, 256)],
                         ids=["cluster", "wide_rows", "many_tokens"])
def test_route_generalised_bitexact(E, top_k, softmax_gates, T, d):
    wl = Workload("route_gen", 14, T, d, 64, E=E, top_k=top_k)
    dev, ora = DeviceLayer(wl), OracleLayer(wl)
    ids, g, logits = jm.jmoe_route(dev.x, dev.w_router, top_k, want_logits=True,
                                   softmax_gates=softmax_gates)
    lo, io, go = oracle.route(ora.x_bits, ora.w_router, top_k, renorm=not softmax_gates)
    assert np.array_equal(logits.cpu().numpy().view(np.uint32), lo.view(np.uint32))
    assert np.array_equal(ids.cpu().numpy(), io)
    gg = g.cpu().numpy().astype(np.float64)
    # fp32 softmax: the denominator sums up to 64 terms, so up to ~64 ulp
    assert np.abs(gg - go).max() <= 4e-6
    if not softmax_gates:
        assert np.abs(gg.sum(axis=1) - 1.0).max() <= gate_sum_bound(top_k)


@pytest.mark.parametrize("E,top_k,T", [(64, 4, 37), (8, 2, 300), (32, 3, 129), (48, 4, 2)],
                         ids=lambda v: str(v))
@pytest.mark.parametrize("path", PATHS)
def test_forward_generalised_routing(E, top_k, T, path):
    wl = Workload("fwd_gen", 15, T, 256, 576, E=E, top_k=top_k)
    dev, ora = DeviceLayer(wl), OracleLayer(wl)
    ids, g = jm.jmoe_route(dev.x, dev.w_router, top_k, softmax_gates=(E == 32))
    out = jm.jmoe_forward(dev.desc(path), dev.x, ids, g)
    torch.cuda.synchronize()
    _, io, go = oracle.route(ora.x_bits, ora.w_router, top_k, renorm=(E != 32))
    assert np.array_equal(ids.cpu().numpy(), io)
    tokens = np.arange(T) if T <= 64 else np.r_[0:8, T - 8:T]
    ref = ora.forward_tokens(tokens, io, go)
    assert_close(bf16_to_f64(out)[tokens], ref, f"E={E} top_k={top_k}")
    assert jm.jmoe_last_error() == jm.JMOE_OK


# ----------------------------------------------------------------------------- RMSNorm prologue


def _bits(t):
    """bf16 bit patterns of a torch bf16 tensor, as uint16."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _norm_inputs(T, d, seed=16):
    x = synth.normal_bf16_gpu(seed, synth.X, 2.0, (T, d))
    g = synth.normal_bf16_gpu(seed + 1, synth.X, 0.25, (d,))
    g = (g.float() + 1.0).to(torch.bfloat16)  # gamma around 1
    return x, g


@pytest.mark.parametrize("T,d", [(37, 256), (1300, 4096), (2, 16384)])
def test_rmsnorm_bitexact(T, d):
    x, g = _norm_inputs(T, d)
    y = jm.jmoe_rmsnorm(x, g, 1e-5)
    torch.cuda.synchronize()
    ref = oracle.rmsnorm(_bits(x), _bits(g), 1e-5)
    assert np.array_equal(_bits(y), ref)


@pytest.mark.parametrize("T,d,E,top_k", [(8, 4096, 16, 2), (37, 256, 64, 4), (1300, 256, 16, 2),
                                         (3, 12288, 16, 2)],
                         ids=["fused", "fused_E64", "many_tokens", "wide_rows"])
def test_rmsnorm_route_bitexact(T, d, E, top_k):
    x, g = _norm_inputs(T, d, seed=17)
    wr = synth.normal_f32_gpu(18, synth.WR, 0.02, (E, d))
    xn, ids, gates, logits = jm.jmoe_rmsnorm_route(x, g, 1e-6, wr, top_k, want_logits=True)
    torch.cuda.synchronize()
    xn_ref = oracle.rmsnorm(_bits(x), _bits(g), 1e-6)
    assert np.array_equal(_bits(xn), xn_ref)
    lo, io, go = oracle.route(xn_ref, wr.cpu().numpy(), top_k)
    assert np.array_equal(logits.cpu().numpy().view(np.uint32), lo.view(np.uint32))
    assert np.array_equal(ids.cpu().numpy(), io)
    assert np.abs(gates.cpu().numpy().astype(np.float64) - go).max() <= 4e-6


@pytest.mark.parametrize("norm", [False, True], ids=["route", "rmsnorm_route"])
def test_layer_graph_matches_eager(norm):
    dev = DeviceLayer(TINY)
    desc = dev.desc(jm.JMOE_PATH_AUTO)
    g = _norm_inputs(1, TINY.d_model)[1] if norm else None
    graph = jm.MoeLayerGraph(desc, dev.w_router, TINY.T, gamma=g, eps=1e-6)
    for seed in (31, 32):
        x = synth.normal_bf16_gpu(seed, synth.X, 1.0, (TINY.T, TINY.d_model))
        out = graph.run(x).clone()
        if norm:
            xn, ids, gates = jm.jmoe_rmsnorm_route(x, g, 1e-6, dev.w_router, TINY.top_k)
        else:
            xn = x
            ids, gates = jm.jmoe_route(x, dev.w_router, TINY.top_k)
        ref = jm.jmoe_forward(desc, xn, ids, gates)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert jm.jmoe_last_error() == jm.JMOE_OK
