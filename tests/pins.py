"""Pins of the CPU oracle against things other than itself.

Each ``pin_*`` function takes an :class:`oracle.Oracle` and raises
``AssertionError`` if the oracle disagrees with exact rational arithmetic,
brute force, a closed form, a textbook special case or an invariant of the
method.  ``test_oracle_pins.py`` runs them against the real oracle;
``test_oracle_mutations.py`` runs them against deliberately broken copies of
the oracle and requires that at least one pin fails for every mutation.

Sources: "Jamba-1.5: Hybrid Transformer-Mamba Models at Scale" (summary page),
section "ExpertsInt8 Quantization (Section 3.1)" steps 1-4 and section "The
Jamba Hybrid Block Structure" (MoE equation); "Jamba: A Hybrid
Transformer-Mamba Language Model" (summary page), section "Mixture-of-Experts
(MoE) in Jamba: Router, Top-K, and Load Balancing" (router softmax, top-K,
renormalised weighted sum) and its layer list (SwiGLU MLP experts).
"""
from __future__ import annotations

import itertools
import json
import os
from fractions import Fraction

import numpy as np

import synth
from exact import (bf16_bits, bf16_value, exact_to_bf16_bits, fr, round_f32_to_bf16_bits,
                   round_half_even, to_fp32)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------------------------------- helpers


def _rand_bf16(seed, tensor, sigma, shape):
    return synth.normal_bf16_bits(seed, tensor, sigma, shape)


def _exact_quantize_row(values):
    """s and q of one row by exact rational arithmetic (the reading stated in
    the golden file): s = fp32(absmax/127), q = rne(fp32(w/s)), clamp +-127."""
    w = [fr(v) for v in values]
    amax = max(abs(v) for v in w)
    if amax == 0:
        return np.float32(0.0), [0] * len(w)
    s = to_fp32(amax / 127)
    q = []
    for v in w:
        quot = fr(to_fp32(v / fr(s)))
        q.append(max(-127, min(127, round_half_even(quot))))
    return s, q


def _dequant(q, s):
    return q.astype(np.float64) * s.astype(np.float64)[:, None]


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _textbook_mlp(x, wgu, wd):
    """SwiGLU MLP with library matmuls: gate rows first, then up rows."""
    f = wd.shape[1]
    u = x @ wgu.T
    h = _silu(u[:, :f]) * u[:, f:]
    return h @ wd.T


def _tiny_experts(o, seed, E, d, f):
    qg, sg, qd, sd = [], [], [], []
    wgu = _rand_bf16(seed, synth.WGU, 0.02, (E, 2 * f, d))
    wd = _rand_bf16(seed, synth.WD, 0.02, (E, d, f))
    for e in range(E):
        q, s = o.quantize(wgu[e])
        qg.append(q)
        sg.append(s)
        q, s = o.quantize(wd[e])
        qd.append(q)
        sd.append(s)
    return qg, sg, qd, sd


# --------------------------------------------------------------------------- quantisation


def pin_quantize_golden_rows(o):
    """Golden rows: q and s equal the exact-rational reading, element by element."""
    with open(os.path.join(GOLDEN, "quantize_rows.json")) as fh:
        rows = json.load(fh)["rows"]
    for row in rows:
        bits = bf16_bits(np.array(row["values"], dtype=np.float32))[None, :]
        q, s = o.quantize(bits)
        s_ref, q_ref = _exact_quantize_row(bf16_value(bits[0]))
        assert s[0] == s_ref, (row["name"], s[0], s_ref)
        assert list(q[0]) == q_ref, (row["name"], list(q[0]), q_ref)


def pin_quantize_random_exact(o):
    """Random bf16 rows (N(0, 0.02)): every q and s equal the exact-rational value."""
    w = _rand_bf16(11, synth.WGU, 0.02, (24, 96))
    q, s = o.quantize(w)
    vals = bf16_value(w)
    for r in range(w.shape[0]):
        s_ref, q_ref = _exact_quantize_row(vals[r])
        assert s[r] == s_ref, (r, s[r], s_ref)
        assert list(q[r]) == q_ref, r


def pin_quantize_roundtrip_bound(o):
    """|w - q*s| <= s/2 * (1 + 2^-16) for every element; absmax -> +-127."""
    w = _rand_bf16(12, synth.WD, 0.02, (256, 512))
    q, s = o.quantize(w)
    wv = bf16_value(w).astype(np.float64)
    err = np.abs(wv - q.astype(np.float64) * s.astype(np.float64)[:, None])
    bound = s.astype(np.float64)[:, None] / 2 * (1 + 2.0 ** -16)
    assert np.all(err <= bound)
    am = np.argmax(np.abs(wv), axis=1)
    got = q[np.arange(q.shape[0]), am]
    assert np.all(np.abs(got.astype(int)) == 127)
    assert np.all(np.sign(got) == np.sign(wv[np.arange(q.shape[0]), am]))
    assert q.min() >= -127 and q.max() <= 127


def pin_quantize_lossless(o):
    """w = k * 2^-7 with max|k| = 127: s = 2^-7 and q = k exactly."""
    rng = np.random.default_rng(3)
    k = rng.integers(-127, 128, size=(8, 64))
    k[:, 5] = 127
    k[::2, 9] = -127
    q, s = o.quantize(bf16_bits((k * 2.0 ** -7).astype(np.float32)))
    assert np.all(s == np.float32(2.0 ** -7))
    assert np.array_equal(q.astype(np.int64), k)


# --------------------------------------------------------------------------- router


def pin_router_canonical_order(o):
    """The logit is the fp64 sum in the canonical order (32 interleaved partial
    sums, then the halving tree).  Partial sums p0 = 2^60, p16 = -2^60, p1 = 1
    give exactly 1 in that order (a left-to-right sum would give 0)."""
    d = 64
    x = np.zeros(d, dtype=np.float32)
    w = np.zeros((2, d), dtype=np.float32)
    x[0], w[0, 0] = 2.0 ** 30, 2.0 ** 30
    x[16], w[0, 16] = 2.0 ** 30, -(2.0 ** 30)
    x[1], w[0, 1] = 1.0, 1.0
    w[1, 2] = 0.5
    x[2] = 1.0
    l = o.router_logits(bf16_bits(x)[None, :], w)
    assert l[0, 0] == np.float32(1.0), l
    assert l[0, 1] == np.float32(0.5), l


def pin_router_logits_exact(o):
    """Random router logits equal fp32 of the exact rational dot product
    (within one fp32 ulp, the only slack the fp64 sum can leave)."""
    T, d, E = 6, 96, 16
    x = _rand_bf16(21, synth.X, 1.0, (T, d))
    wr = synth.normal_f32(21, synth.WR, 0.02, (E, d))
    bias = np.array([0.25 * (e % 3) for e in range(E)], dtype=np.float32)
    l = o.router_logits(x, wr, bias)
    xv = bf16_value(x)
    for t in range(T):
        for e in range(E):
            exact = sum((fr(xv[t, k]) * fr(wr[e, k]) for k in range(d)), Fraction(0)) + fr(bias[e])
            ref = to_fp32(exact)
            assert abs(float(l[t, e]) - float(ref)) <= abs(float(np.spacing(np.float32(ref)))), (t, e)


def pin_router_bias_exact(o):
    """x = 0: every logit equals its bias exactly."""
    d, E = 64, 16
    wr = synth.normal_f32(5, synth.WR, 0.02, (E, d))
    bias = np.linspace(-3, 3, E).astype(np.float32)
    l = o.router_logits(np.zeros((3, d), dtype=np.uint16), wr, bias)
    assert np.array_equal(l, np.tile(bias, (3, 1)))


def _topk_bruteforce(l, k):
    """All ordered k-tuples; the winner is the lexicographically largest key
    sequence (logit, then lower index)."""
    E = len(l)
    best, best_key = None, None
    for combo in itertools.permutations(range(E), k):
        key = tuple(x for e in combo for x in (float(l[e]), -e))
        if best_key is None or key > best_key:
            best, best_key = combo, key
    return list(best)


def pin_topk_bruteforce(o):
    """Top-2 (and top-1, top-3; top-4 of 8) ids equal brute force over all
    ordered tuples."""
    rng = np.random.default_rng(7)
    for k, E in ((1, 16), (2, 16), (3, 16), (4, 8)):
        l = rng.standard_normal((40, E)).astype(np.float32)
        l[:5, 4] = l[:5, E - 5] = 3.0  # exact ties at the top
        l[5:10, 2] = l[5:10, E - 7] = l[5:10, E - 3] = 2.5  # three-way ties
        ids, _ = o.topk_gates(l, k)
        for t in range(l.shape[0]):
            assert list(ids[t]) == _topk_bruteforce(l[t], k), (k, t)


def pin_topk_wide_stable_sort(o):
    """64 experts, top-4: the ids are the first four of a stable descending
    sort of the logits (equal logits keep ascending index order)."""
    rng = np.random.default_rng(17)
    l = rng.integers(-6, 7, size=(200, 64)).astype(np.float32) / 2  # many exact ties
    ids, _ = o.topk_gates(l, 4)
    ref = np.argsort(-l, axis=1, kind="stable")[:, :4]
    assert np.array_equal(ids, ref)


def pin_softmax_gates(o):
    """Plain softmax gates (no renormalisation).  Closed forms: with two
    experts and top-1 the gate is the logistic function of the logit gap;
    with every expert selected the gates sum to 1 and g_i / g_j =
    exp(l_i - l_j); and plain = renormalised x (sum of the plain gates)."""
    rng = np.random.default_rng(18)
    l2 = (rng.standard_normal((64, 2)) * 3).astype(np.float32)
    ids, g = o.topk_gates(l2, 1, renorm=False)
    lo = l2[np.arange(64), 1 - ids[:, 0]].astype(np.float64)
    ls = l2[np.arange(64), ids[:, 0]].astype(np.float64)
    assert np.allclose(g[:, 0], 1.0 / (1.0 + np.exp(lo - ls)), rtol=0, atol=1e-15)
    l4 = (rng.standard_normal((64, 4)) * 2).astype(np.float32)
    ids4, g4 = o.topk_gates(l4, 4, renorm=False)
    assert np.allclose(g4.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    li = np.take_along_axis(l4, ids4, axis=1).astype(np.float64)
    assert np.allclose(g4[:, 1:] / g4[:, :1], np.exp(li[:, 1:] - li[:, :1]), rtol=1e-14, atol=0)
    l16 = (rng.standard_normal((64, 16)) * 2).astype(np.float32)
    for k in (1, 2, 4):
        idp, gp = o.topk_gates(l16, k, renorm=False)
        idr, gr = o.topk_gates(l16, k, renorm=True)
        assert np.array_equal(idp, idr)
        assert np.allclose(gp, gr * gp.sum(axis=1, keepdims=True), rtol=1e-15, atol=0)
        assert np.all(gp.sum(axis=1) <= 1.0 + 1e-15)


def pin_topk_tie_identical_rows(o):
    """Identical router rows 3 and 7 give identical logits; when both are in
    the top-2, expert 3 is listed first (ties go to the lower index)."""
    d, E = 64, 16
    wr = synth.normal_f32(9, synth.WR, 0.02, (E, d))
    wr[7] = wr[3]
    bias = np.zeros(E, dtype=np.float32)
    bias[3] = bias[7] = 4.0
    x = _rand_bf16(9, synth.X, 1.0, (10, d))
    _, ids, g = o.route(x, wr, 2, bias)
    assert np.all(ids[:, 0] == 3) and np.all(ids[:, 1] == 7)
    assert np.all(g == 0.5)


def pin_gates(o):
    """Gates: renormalised softmax of the selected logits.  Closed forms:
    top-2 g1 = 1/(1 + exp(l2 - l1)), g1 + g2 = 1; top-1 g = 1; E = 1 g = 1."""
    rng = np.random.default_rng(8)
    l = (rng.standard_normal((64, 16)) * 2).astype(np.float32)
    ids, g = o.topk_gates(l, 2)
    l1 = l[np.arange(64), ids[:, 0]].astype(np.float64)
    l2 = l[np.arange(64), ids[:, 1]].astype(np.float64)
    assert np.allclose(g[:, 0], 1.0 / (1.0 + np.exp(l2 - l1)), rtol=0, atol=1e-15)
    assert np.allclose(g.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    assert np.all(g[:, 0] >= g[:, 1])
    ids1, g1 = o.topk_gates(l, 1)
    assert np.all(g1 == 1.0)
    _, ge = o.topk_gates(l[:, :1], 1)
    assert np.all(ge == 1.0)
    # large logits (activations reach thousands in these models): the gates
    # still follow the closed form, g1 = 1/(1 + e^-1) for a gap of 1
    big = np.full((2, 16), 900.0, dtype=np.float32)
    big[:, 3] = 1001.0
    big[:, 12] = 1000.0
    idsb, gb = o.topk_gates(big, 2)
    assert np.array_equal(idsb, [[3, 12], [3, 12]])
    assert np.allclose(gb[:, 0], 1.0 / (1.0 + np.exp(-1.0)), rtol=1e-15, atol=0)
    # top-3: each gate is its softmax probability over the selected set
    ids3, g3 = o.topk_gates(l, 3)
    sel = np.take_along_axis(l.astype(np.float64), ids3, axis=1)
    ref = np.exp(sel) / np.exp(sel).sum(axis=1, keepdims=True)
    assert np.allclose(g3, ref, rtol=1e-13, atol=0)


def pin_skew_fraction(o):
    """Bias +2.0 on experts 0 and 1 with Large-like logits (d = 8192) sends
    roughly 40 % of the assignments to them (about 12.5 % without bias)."""
    T, d, E = 256, 8192, 16
    x = _rand_bf16(30, synth.X, 1.0, (T, d))
    wr = synth.normal_f32(30, synth.WR, 0.02, (E, d))
    bias = np.array([2.0 if e < 2 else 0.0 for e in range(E)], dtype=np.float32)
    _, ids, _ = o.route(x, wr, 2, bias)
    frac = float(np.isin(ids, [0, 1]).mean())
    assert 0.33 <= frac <= 0.47, frac
    _, ids0, _ = o.route(x, wr, 2, None)
    frac0 = float(np.isin(ids0, [0, 1]).mean())
    assert frac0 < 0.2, frac0


# --------------------------------------------------------------------------- permutation


def pin_permute_bruteforce(o):
    """Stable sort of the assignments by expert, by Python's sorted()."""
    rng = np.random.default_rng(4)
    for T, k, E in [(37, 2, 16), (5, 1, 4), (64, 2, 16), (1, 2, 16), (0, 2, 16), (50, 3, 8)]:
        ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
        if T > 3:
            ids[:, 0] = np.minimum(ids[:, 0], 3)  # skew: crowd a few experts
        offsets, perm, inv = o.permute(ids, E)
        flat = ids.reshape(-1)
        ref = sorted(range(T * k), key=lambda a: flat[a])
        assert list(perm) == ref
        counts = np.bincount(flat, minlength=E)
        assert list(offsets) == [0] + list(np.cumsum(counts))
        assert np.array_equal(inv[perm], np.arange(T * k))


# --------------------------------------------------------------------------- experts + combine


def pin_dense_equals_textbook(o):
    """E = 1, top-1: the layer is the textbook SwiGLU MLP on the dequantised
    weights w = q*s (numpy matmuls), gate rows first."""
    T, d, f = 7, 64, 96
    x = _rand_bf16(40, synth.X, 1.0, (T, d))
    qg, sg, qd, sd = _tiny_experts(o, 40, 1, d, f)
    xv = bf16_value(x).astype(np.float64)
    ref = _textbook_mlp(xv, _dequant(qg[0], sg[0]), _dequant(qd[0], sd[0]))
    out = o.mlp_forward(x, qg[0], sg[0], qd[0], sd[0])
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    ids = np.zeros((T, 1), dtype=np.int32)
    out2 = o.moe_forward(x, ids, np.ones((T, 1)), qg, sg, qd, sd)
    assert np.allclose(out2, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # the convention is pinned: swapping the gate and up halves changes the result
    swapped = np.concatenate([qg[0][f:], qg[0][:f]])
    sw_s = np.concatenate([sg[0][f:], sg[0][:f]])
    ref_sw = _textbook_mlp(xv, _dequant(swapped, sw_s), _dequant(qd[0], sd[0]))
    assert not np.allclose(ref_sw, ref, rtol=1e-3)


def pin_moe_equals_weighted_textbook(o):
    """MoE output = sum_j g_j * textbook_MLP_{e_j}(x) with the oracle's routing."""
    T, d, f, E = 9, 64, 96, 16
    x = _rand_bf16(41, synth.X, 1.0, (T, d))
    wr = synth.normal_f32(41, synth.WR, 0.02, (E, d))
    qg, sg, qd, sd = _tiny_experts(o, 41, E, d, f)
    _, ids, g = o.route(x, wr, 2)
    out = o.moe_forward(x, ids, g, qg, sg, qd, sd)
    xv = bf16_value(x).astype(np.float64)
    ref = np.zeros((T, d))
    for t in range(T):
        for j in range(2):
            e = ids[t, j]
            ref[t] += g[t, j] * _textbook_mlp(xv[t:t + 1], _dequant(qg[e], sg[e]),
                                              _dequant(qd[e], sd[e]))[0]
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def pin_zero_input(o):
    """x = 0 gives exactly 0 (silu(0) * 0 = 0)."""
    T, d, f, E = 4, 64, 96, 16
    qg, sg, qd, sd = _tiny_experts(o, 42, E, d, f)
    wr = synth.normal_f32(42, synth.WR, 0.02, (E, d))
    x = np.zeros((T, d), dtype=np.uint16)
    _, ids, g = o.route(x, wr, 2)
    assert np.array_equal(ids, np.tile([0, 1], (T, 1)))  # all logits 0: ties -> 0, 1
    assert np.all(g == 0.5)
    assert np.all(o.moe_forward(x, ids, g, qg, sg, qd, sd) == 0.0)


def pin_forced_routing(o):
    """All tokens to expert 5 (twice, gates 0.25/0.75) equals the dense MLP on
    expert 5's weights; one token split over two experts combines linearly."""
    T, d, f, E = 6, 64, 96, 16
    x = _rand_bf16(43, synth.X, 1.0, (T, d))
    qg, sg, qd, sd = _tiny_experts(o, 43, E, d, f)
    dense = o.mlp_forward(x, qg[5], sg[5], qd[5], sd[5])
    ids = np.full((T, 2), 5, dtype=np.int32)
    g = np.tile([0.25, 0.75], (T, 1))
    out = o.moe_forward(x, ids, g, qg, sg, qd, sd)
    assert np.allclose(out, dense, rtol=1e-13, atol=1e-13 * np.abs(dense).max())
    d9 = o.mlp_forward(x, qg[9], sg[9], qd[9], sd[9])
    ids2 = np.tile([5, 9], (T, 1)).astype(np.int32)
    g2 = np.tile([0.3, 0.7], (T, 1))
    out2 = o.moe_forward(x, ids2, g2, qg, sg, qd, sd)
    assert np.allclose(out2, 0.3 * dense + 0.7 * d9, rtol=1e-12,
                       atol=1e-12 * np.abs(dense).max())


def pin_relabel_and_token_order(o):
    """Relabelling the experts (router rows and weights together) leaves the
    output unchanged; permuting the tokens permutes the output rows."""
    T, d, f, E = 12, 64, 96, 16
    x = _rand_bf16(44, synth.X, 1.0, (T, d))
    wr = synth.normal_f32(44, synth.WR, 0.02, (E, d))
    qg, sg, qd, sd = _tiny_experts(o, 44, E, d, f)
    _, ids, g = o.route(x, wr, 2)
    out = o.moe_forward(x, ids, g, qg, sg, qd, sd)
    pi = np.random.default_rng(1).permutation(E)  # new label of old expert e is pi[e]
    inv = np.argsort(pi)
    wr2 = wr[inv]
    _, ids2, g2 = o.route(x, wr2, 2)
    out2 = o.moe_forward(x, ids2, g2, [qg[i] for i in inv], [sg[i] for i in inv],
                         [qd[i] for i in inv], [sd[i] for i in inv])
    assert np.array_equal(pi[ids], ids2)
    # the softmax normaliser is summed in a different expert order, so gates
    # (and the output) agree to fp64 rounding rather than bit for bit
    assert np.allclose(g, g2, rtol=1e-14, atol=0)
    assert np.allclose(out, out2, rtol=1e-13, atol=1e-13 * np.abs(out).max())
    tp = np.random.default_rng(2).permutation(T)
    _, ids3, g3 = o.route(x[tp], wr, 2)
    out3 = o.moe_forward(x[tp], ids3, g3, qg, sg, qd, sd)
    assert np.array_equal(out3, out[tp])


def pin_lossless_equals_bf16_mlp(o):
    """Weights already on the INT8 grid (k * 2^-7) quantise losslessly, so the
    INT8 layer equals the unquantised BF16 MLP (numpy fp64 on bf16 values)."""
    T, d, f = 5, 64, 96
    rng = np.random.default_rng(6)
    kg = rng.integers(-127, 128, size=(2 * f, d))
    kg[:, 0] = 127
    kd = rng.integers(-127, 128, size=(d, f))
    kd[:, 0] = -127
    wg = (kg * 2.0 ** -7).astype(np.float32)
    wd = (kd * 2.0 ** -7).astype(np.float32)
    x = _rand_bf16(45, synth.X, 1.0, (T, d))
    qg, sg = o.quantize(bf16_bits(wg))
    qd, sd = o.quantize(bf16_bits(wd))
    out = o.mlp_forward(x, qg, sg, qd, sd)
    ref = _textbook_mlp(bf16_value(x).astype(np.float64), wg.astype(np.float64),
                        wd.astype(np.float64))
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def pin_silu_closed_form(o):
    """One channel, identity-like weights: out = s_d*q_d * silu(u_g) * u_u with
    u known exactly; silu(z) = z * sigmoid(z) at z = 0, +-1, 3."""
    d, f = 4, 1
    for z in (0.0, 1.0, -1.0, 3.0):
        # x = [z, 1, 0, 0]; gate row picks x0, up row picks x1 (both *1 after scale 1/127*127)
        x = bf16_bits(np.array([[z, 1.0, 0.0, 0.0]], dtype=np.float32))
        wg = np.array([[1.0, 0, 0, 0], [0, 1.0, 0, 0]], dtype=np.float32)
        wd = np.array([[1.0], [0.5], [0.0], [-2.0]], dtype=np.float32)
        qg, sg = o.quantize(bf16_bits(wg))
        qd, sd = o.quantize(bf16_bits(wd))
        out = o.mlp_forward(x, qg, sg, qd, sd)[0]
        ug = float(fr(sg[0]) * 127) * z
        uu = float(fr(sg[1]) * 127) * 1.0
        h = ug / (1.0 + np.exp(-ug)) * uu
        ref = np.array([float(fr(sd[m]) * int(qd[m, 0])) * h for m in range(4)])
        assert np.allclose(out, ref, rtol=1e-14, atol=1e-300), (z, out, ref)


def _rmsnorm_exact(x_bits, g_bits, eps):
    """RMSNorm to ~60 digits (Fractions, Decimal square root), rounded once to
    bf16: the value the oracle must hit unless it lies within a few fp64 ulps
    of a bf16 rounding boundary."""
    import decimal
    from fractions import Fraction

    ctx = decimal.Context(prec=60)
    x = [fr(v) for v in bf16_value(x_bits)]
    g = [fr(v) for v in bf16_value(g_bits)]
    mean = sum(v * v for v in x) / len(x) + fr(np.float32(eps))
    rs = ctx.divide(decimal.Decimal(1), ctx.sqrt(ctx.divide(decimal.Decimal(mean.numerator),
                                                            decimal.Decimal(mean.denominator))))
    r = Fraction(rs)
    return np.array([exact_to_bf16_bits(xv * r * gv) for xv, gv in zip(x, g)], dtype=np.uint16)


def pin_rmsnorm_exact(o):
    """RMSNorm equals the exact value rounded once to bf16, for a typical eps
    and for a large eps on small activations (where dropping eps shows)."""
    rng = np.random.default_rng(21)
    for sigma, eps in ((1.0, 1e-6), (0.4, 0.5)):
        x = round_f32_to_bf16_bits((rng.standard_normal((6, 96)) * sigma).astype(np.float32))
        g = round_f32_to_bf16_bits((1.0 + 0.25 * rng.standard_normal(96)).astype(np.float32))
        y = o.rmsnorm(x, g, eps)
        for t in range(x.shape[0]):
            assert np.array_equal(y[t], _rmsnorm_exact(x[t], g, eps)), (sigma, eps, t)


def pin_rmsnorm_invariants(o):
    """Bitwise: y(-x) = -y(x); with eps = 0, y(2^m x) = y(x); doubling gamma
    doubles y; a constant row with gamma = 1 and eps = 0 normalises to +-1."""
    rng = np.random.default_rng(22)
    x = round_f32_to_bf16_bits(rng.standard_normal((8, 128)).astype(np.float32))
    g = round_f32_to_bf16_bits((0.5 + rng.random(128)).astype(np.float32))
    y = o.rmsnorm(x, g, 0.0)
    assert np.array_equal(o.rmsnorm(x ^ np.uint16(0x8000), g, 0.0), y ^ np.uint16(0x8000))
    x32 = bf16_bits(bf16_value(x) * 32.0)
    assert np.array_equal(o.rmsnorm(x32, g, 0.0), y)
    g2 = bf16_bits(bf16_value(g) * 2.0)
    assert np.array_equal(bf16_value(o.rmsnorm(x, g2, 0.0)), bf16_value(y) * 2.0)
    c = np.full((3, 64), 0, dtype=np.uint16)
    c[0], c[1], c[2] = bf16_bits([3.0])[0], bf16_bits([-0.125])[0], bf16_bits([1.5])[0]
    ones = bf16_bits(np.ones(64))
    yc = bf16_value(o.rmsnorm(c, ones, 0.0))
    assert np.all(yc[0] == 1.0) and np.all(yc[1] == -1.0) and np.all(yc[2] == 1.0)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
