"""Every plausible single mistake in the oracle is caught by at least one pin.

Each case copies ``oracle/oracle.c``, plants one mistake (on the CPU, in the
copy only), compiles it, and runs every pin of ``pins.py`` against it.  The
test passes when at least one pin rejects the broken copy.
"""
import os

import pytest

import oracle
import pins

MUTATIONS = [
    # quantisation
    ("reciprocal_multiply", "rintf(bf16_to_f32(w[k]) / s)", "rintf(bf16_to_f32(w[k]) * (1.0f / s))"),
    ("round_half_away", "rintf(bf16_to_f32(w[k]) / s)", "roundf(bf16_to_f32(w[k]) / s)"),
    ("truncate_not_round", "rintf(bf16_to_f32(w[k]) / s)", "truncf(bf16_to_f32(w[k]) / s)"),
    ("scale_by_128", "float s = amax / 127.0f;", "float s = amax / 128.0f;"),
    # router
    ("sequential_partials",
     "for (int o = 16; o >= 1; o /= 2)\n                for (int j = 0; j < o; ++j) p[j] = p[j] + p[j + o];",
     "for (int j = 1; j < 32; ++j) p[0] = p[0] + p[j];"),
    ("bias_dropped", "double b = bias_or_null ? (double)bias_or_null[e] : 0.0;", "double b = 0.0;"),
    ("logit_fp32_accumulate", "p[j] += (double)bf16_to_f32(x[k]) * (double)w[k];",
     "p[j] = (float)(p[j] + (float)(bf16_to_f32(x[k]) * w[k]));"),
    # top-k and gates
    ("ties_to_higher_index", "if (best < 0 || l[e] > l[best]) best = e;",
     "if (best < 0 || l[e] >= l[best]) best = e;"),
    ("gates_not_renormalised", "gates[t * top_k + j] = renorm ? p[chosen[j]] / sel : p[chosen[j]];",
     "gates[t * top_k + j] = p[chosen[j]];"),
    ("softmax_gates_renormalised",
     "gates[t * top_k + j] = renorm ? p[chosen[j]] / sel : p[chosen[j]];",
     "gates[t * top_k + j] = p[chosen[j]] / sel;"),
    ("softmax_gates_over_selection_only", "for (int e = 0; e < E; ++e) p[e] /= z;",
     "for (int e = 0; e < E; ++e) p[e] /= z;\n        if (!renorm) { double zs = 0.0; for (int j = 0; j < top_k; ++j) zs += p[chosen[j]]; for (int e = 0; e < E; ++e) p[e] /= zs; }"),
    ("topk_allows_repeats", "if (taken) continue;", "(void)taken;"),
    ("softmax_missing_max_shift", "p[e] = exp((double)l[e] - m);", "p[e] = exp((double)l[e]);"),
    # RMSNorm ahead of the router
    ("rmsnorm_eps_dropped", "1.0 / sqrt(p[0] / (double)d + (double)eps)", "1.0 / sqrt(p[0] / (double)d)"),
    ("rmsnorm_sum_not_mean", "1.0 / sqrt(p[0] / (double)d + (double)eps)",
     "1.0 / sqrt(p[0] + (double)eps)"),
    ("rmsnorm_no_sqrt", "1.0 / sqrt(p[0] / (double)d + (double)eps)",
     "1.0 / (p[0] / (double)d + (double)eps)"),
    ("rmsnorm_gamma_ignored", "((double)bf16_to_f32(x[k]) * r) *\n                                                 (double)bf16_to_f32(gamma_bf16[k])",
     "((double)bf16_to_f32(x[k]) * r)"),
    # permutation
    ("permute_reverse_order", "for (int64_t a = 0; a < A; ++a) {\n        int32_t pos",
     "for (int64_t a = A - 1; a >= 0; --a) {\n        int32_t pos"),
    # experts and combine
    ("gate_up_swapped", "double g = u[n];", "double g = u[f + n];"),
    ("silu_sign", "double silu = g / (1.0 + exp(-g));", "double silu = g / (1.0 + exp(g));"),
    ("relu_not_silu", "double silu = g / (1.0 + exp(-g));", "double silu = g > 0 ? g : 0.0;"),
    ("down_scale_dropped", "acc += h[n] * ((double)qr[n] * (double)s_d[m]);",
     "acc += h[n] * (double)qr[n];"),
    ("gateup_scale_dropped", "acc += xd[k] * ((double)qr[k] * (double)s_gu[n]);",
     "acc += xd[k] * (double)qr[k];"),
    ("gate_not_applied", "out[t * d + m] += g * y[m];", "out[t * d + m] += y[m];"),
    ("combine_overwrites", "out[t * d + m] += g * y[m];", "out[t * d + m] = g * y[m];"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(name, old, new, tmp_path):
    with open(oracle.SOURCE) as fh:
        src = fh.read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutated = tmp_path / f"oracle_{name}.c"
    mutated.write_text(src.replace(old, new))
    so = str(tmp_path / f"liboracle_{name}.so")
    oracle.compile_oracle(str(mutated), so)
    broken = oracle.Oracle(so)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(broken)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin rejects the mutation {name}"
    assert os.path.exists(so)
